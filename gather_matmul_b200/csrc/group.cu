// Token-index metadata: group-by-slot (stable counting sort) and the work
// lists the per-token kernels consume.
//
// The token-index tensor is built on the host and moved to the device once
// per batch ("[Hardware][TPU][V1] Better tpu multilora compilation", review
// thread on moving the token LoRA indices to the device); everything after
// that happens here, on the device, without a host round trip.  Grouping
// tokens by slot is what lets one CTA stage an adapter's weights once and use
// them for every token of that adapter, instead of the per-token gather whose
// copies made the PyTorch baseline slow (same page, discussion of the
// index_select copies).
#include "common.cuh"
#include "internal.h"

namespace lora {

namespace {

constexpr int kGroupThreads = 1024;
constexpr int kGroupWarps = kGroupThreads / 32;

// Exclusive scan of n <= 2 * kGroupThreads ints in shared memory, in place;
// returns the total.  Must be called by all threads of the block.
__device__ int block_exclusive_scan(int* a, int n, int* warp_tmp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int i0 = 2 * tid, i1 = 2 * tid + 1;
  int v0 = i0 < n ? a[i0] : 0;
  int v1 = i1 < n ? a[i1] : 0;
  int s = v0 + v1;
  int inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) warp_tmp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kGroupWarps ? warp_tmp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    warp_tmp[32 + lane] = wi - w;   // exclusive prefix of warp totals
    if (lane == 31) warp_tmp[64] = wi;
  }
  __syncthreads();
  int excl = warp_tmp[32 + warp] + inc - s;
  if (i0 < n) a[i0] = excl;
  if (i1 < n) a[i1] = excl + v0;
  int total = warp_tmp[64];
  __syncthreads();
  return total;
}

// One CTA.  Shared memory: cnt[kGroupWarps][K], tot[K], base[K], ni[K],
// plus 65 ints of scan scratch, with K = S + 1 keys (slot S = no adapter).
__global__ void __launch_bounds__(kGroupThreads, 1)
group_kernel(int T, int S, const int32_t* __restrict__ idx, char* __restrict__ meta) {
  extern __shared__ int smem[];
  const int K = S + 1;
  int* cnt = smem;                          // [warp][key]
  int* tot = cnt + kGroupWarps * K;         // count per key
  int* base = tot + K;                      // first position per key
  int* ni = base + K;                       // items per key, then item offsets
  int* scratch = ni + K;                    // 65 ints

  MetaLayout L(T, S);
  MetaHeader* hdr = reinterpret_cast<MetaHeader*>(meta);
  int* slot_off = reinterpret_cast<int*>(meta + L.off_slot);
  int* perm = reinterpret_cast<int*>(meta + L.off_perm);
  int4* items = reinterpret_cast<int4*>(meta + L.off_items);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kGroupWarps * K; i += kGroupThreads) cnt[i] = 0;
  __syncthreads();

  // Each warp owns one contiguous range of tokens, walked 32 at a time.
  const int chunk = (((T + kGroupWarps - 1) / kGroupWarps) + 31) & ~31;
  const int beg = warp * chunk;
  const int end = min(T, beg + chunk);
  int bad = 0;
  for (int b = beg; b < end; b += 32) {
    int t = b + lane;
    bool valid = t < end;
    int v = valid ? idx[t] : -1;
    if (valid && (v < -1 || v >= S)) ++bad;
    int key = valid ? ((v >= 0 && v < S) ? v : S) : -1;
    unsigned peers = __match_any_sync(0xffffffffu, key);
    if (valid && lane == __ffs(peers) - 1) cnt[warp * K + key] += __popc(peers);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if (lane == 0 && bad) atomicAdd(&hdr->bad_index, bad);
  __syncthreads();

  for (int k = tid; k < K; k += kGroupThreads) {
    int s = 0;
    for (int w = 0; w < kGroupWarps; ++w) s += cnt[w * K + k];
    tot[k] = s;
    base[k] = s;
    ni[k] = (s + kItemTokens - 1) / kItemTokens;
  }
  __syncthreads();
  // K <= LORA_MAX_SLOTS + 1 <= 2 * kGroupThreads
  block_exclusive_scan(base, K, scratch);
  int n_items = block_exclusive_scan(ni, K, scratch);

  for (int k = tid; k < K; k += kGroupThreads) {
    slot_off[k] = base[k];
    int run = base[k];
    for (int w = 0; w < kGroupWarps; ++w) {   // per-(warp, key) start positions
      int c = cnt[w * K + k];
      cnt[w * K + k] = run;
      run += c;
    }
    int it0 = ni[k];
    int n = tot[k];
    for (int j = 0; j * kItemTokens < n; ++j) {
      int b0 = base[k] + j * kItemTokens;
      int e0 = min(base[k] + n, b0 + kItemTokens);
      items[it0 + j] = make_int4(k < S ? k : -1, b0, e0, 0);
    }
  }
  if (tid == 0) {
    slot_off[K] = T;
    hdr->n_items = n_items;
    hdr->n_active = base[S];
    hdr->T = T;
    hdr->S = S;
  }
  __syncthreads();

  // Stable scatter: the same walk; a token's rank among equal keys of its
  // 32-token step comes from the match mask.
  for (int b = beg; b < end; b += 32) {
    int t = b + lane;
    bool valid = t < end;
    int v = valid ? idx[t] : -1;
    int key = valid ? ((v >= 0 && v < S) ? v : S) : -1;
    unsigned peers = __match_any_sync(0xffffffffu, key);
    int pos = 0;
    if (valid) pos = cnt[warp * K + key] + __popc(peers & lanemask_lt());
    __syncwarp();
    if (valid) {
      perm[pos] = t;
      if (lane == __ffs(peers) - 1) cnt[warp * K + key] += __popc(peers);
    }
    __syncwarp();
  }
}

// Work list for segments: each segment becomes ceil(len / 16) items with the
// segment's adapter, tokens addressed directly.  Malformed lists (first != 0,
// last != T, decreasing) produce no items and are counted as bad.
__global__ void __launch_bounds__(kGroupThreads, 1)
segment_items_kernel(int T, int S, int n_seg, const int32_t* __restrict__ seg_starts,
                     const int32_t* __restrict__ seg_adapter, char* __restrict__ meta) {
  __shared__ int tile[2 * kGroupThreads];
  __shared__ int scratch[65];
  __shared__ int s_bad, s_carry;
  MetaLayout L(T, S);
  MetaHeader* hdr = reinterpret_cast<MetaHeader*>(meta);
  int4* items = reinterpret_cast<int4*>(meta + L.off_items);
  const int tid = threadIdx.x;
  if (tid == 0) { s_bad = 0; s_carry = 0; }
  __syncthreads();
  int bad = 0, bad_adapter = 0;
  if (tid == 0 && (seg_starts[0] != 0 || seg_starts[n_seg] != T)) bad = 1;
  for (int s = tid; s < n_seg; s += kGroupThreads) {
    int a = seg_starts[s], b = seg_starts[s + 1];
    if (b < a || a < 0 || b > T) bad = 1;
    int ad = seg_adapter[s];
    if (ad < -1 || ad >= S) bad_adapter += b > a ? b - a : 0;
  }
  if (bad) atomicOr(&s_bad, 1);
  if (bad_adapter) atomicAdd(&hdr->bad_index, bad_adapter);
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      atomicAdd(&hdr->bad_meta, 1);
      hdr->n_items = 0;
      hdr->T = T;
      hdr->S = S;
    }
    return;
  }
  // chunked scan over segments of their item counts
  for (int s0 = 0; s0 < n_seg; s0 += 2 * kGroupThreads) {
    int n = min(n_seg - s0, 2 * kGroupThreads);
    for (int k = tid; k < n; k += kGroupThreads) {
      int len = seg_starts[s0 + k + 1] - seg_starts[s0 + k];
      tile[k] = (len + kItemTokens - 1) / kItemTokens;
    }
    __syncthreads();
    int total = block_exclusive_scan(tile, n, scratch);
    int carry = s_carry;
    for (int k = tid; k < n; k += kGroupThreads) {
      int s = s0 + k;
      int a = seg_starts[s], b = seg_starts[s + 1];
      int ad = seg_adapter[s];
      int slot = (ad >= 0 && ad < S) ? ad : -1;
      int it0 = carry + tile[k];
      for (int j = 0; a + j * kItemTokens < b; ++j) {
        int b0 = a + j * kItemTokens;
        items[it0 + j] = make_int4(slot, b0, min(b, b0 + kItemTokens), kItemDirect);
      }
    }
    __syncthreads();
    if (tid == 0) s_carry = carry + total;
    __syncthreads();
  }
  if (tid == 0) {
    hdr->n_items = s_carry;
    hdr->T = T;
    hdr->S = S;
  }
}

}  // namespace

size_t group_smem_bytes(int S) {
  return sizeof(int) * ((size_t)(kGroupWarps + 3) * (S + 1) + 65);
}

cudaError_t launch_group(int T, int S, const int32_t* idx, void* meta, cudaStream_t st) {
  size_t smem = group_smem_bytes(S);
  cudaError_t e = cudaFuncSetAttribute(group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  group_kernel<<<1, kGroupThreads, smem, st>>>(T, S, idx, static_cast<char*>(meta));
  return counted_launch(cudaGetLastError());
}

cudaError_t launch_segment_items(int T, int S, int n_seg, const int32_t* seg_starts,
                                 const int32_t* seg_adapter, void* meta, cudaStream_t st) {
  segment_items_kernel<<<1, kGroupThreads, 0, st>>>(T, S, n_seg, seg_starts, seg_adapter,
                                                    static_cast<char*>(meta));
  return counted_launch(cudaGetLastError());
}

}  // namespace lora
