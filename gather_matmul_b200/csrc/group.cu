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
#include "ptx.cuh"

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

// Exclusive scans of two arrays of n <= 2 * kGroupThreads ints in shared
// memory, in place, sharing their barriers; the totals go to *ta and *tb.
// Must be called by all threads of the block.
__device__ void block_exclusive_scan2(int* a, int* b, int n, int* warp_tmp, int* ta, int* tb) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = 2 * tid, i1 = 2 * tid + 1;
  const int a0 = i0 < n ? a[i0] : 0, a1 = i1 < n ? a[i1] : 0;
  const int b0 = i0 < n ? b[i0] : 0, b1 = i1 < n ? b[i1] : 0;
  const int sa = a0 + a1, sb = b0 + b1;
  int ia = sa, ib = sb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ua = __shfl_up_sync(0xffffffffu, ia, o);
    const int ub = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += ua;
      ib += ub;
    }
  }
  if (lane == 31) {
    warp_tmp[warp] = ia;
    warp_tmp[32 + warp] = ib;
  }
  __syncthreads();
  if (warp == 0) {
    const int wa = lane < kGroupWarps ? warp_tmp[lane] : 0;
    const int wb = lane < kGroupWarps ? warp_tmp[32 + lane] : 0;
    int xa = wa, xb = wb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ua = __shfl_up_sync(0xffffffffu, xa, o);
      const int ub = __shfl_up_sync(0xffffffffu, xb, o);
      if (lane >= o) {
        xa += ua;
        xb += ub;
      }
    }
    warp_tmp[64 + lane] = xa - wa;     // exclusive prefixes of the warp totals
    warp_tmp[96 + lane] = xb - wb;
    if (lane == 31) {
      *ta = xa;
      *tb = xb;
    }
  }
  __syncthreads();
  const int ea = warp_tmp[64 + warp] + ia - sa, eb = warp_tmp[96 + warp] + ib - sb;
  if (i0 < n) {
    a[i0] = ea;
    b[i0] = eb;
  }
  if (i1 < n) {
    a[i1] = ea + a0;
    b[i1] = eb + b0;
  }
  __syncthreads();
}

// Generation barrier of the grouping kernel's CTAs, kept in the workspace
// header.  Thread 0 of each CTA calls it once its CTA's histogram row is
// written and fenced.  The last CTA to arrive resets the count and opens the
// next generation, so the barrier is reusable whatever the CTA count of the
// next launch.  The wait is bounded (about one second): on a timeout it
// returns false and the caller records an error instead of hanging.
__device__ bool group_barrier(MetaHeader* hdr, int nb) {
  volatile int* gen = &hdr->bar_gen;
  const int g0 = *gen;
  __threadfence();
  if (atomicAdd(&hdr->bar_count, 1) == nb - 1) {
    atomicExch(&hdr->bar_count, 0);
    __threadfence();
    atomicAdd(&hdr->bar_gen, 1);
    return true;
  }
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  while (*gen == g0) {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > 1000000000ull) return false;
    __nanosleep(200);
  }
  __threadfence();
  return true;
}

constexpr int kLoadBatch = 8;   // indices a lane has in flight at once

// Per-(key, warp) counts are kept key-major with a pitch of 33 ints, so the
// counts of one key across the 32 warps are one conflict-free row that a
// warp scans with shuffles.
constexpr int kCntPitch = kGroupWarps + 1;

// group_ctas(T) CTAs, each over a contiguous chunk of the tokens; each warp
// over a contiguous part of its CTA's chunk, so CTA, warp and lane order is
// token order and the scatter is stable.  Shared memory: cnt[K][33],
// tot[K], base[K], pre[K], ni[K] and 130 ints of scan scratch, K = S + 1
// keys (key S = no adapter).
//   1. per-warp counts of each key (warp match_any); one warp per key scans
//      the key's 32 warp counts (each warp's offset inside the CTA) and
//      writes the CTA's total into its row of the workspace histogram;
//   2. barrier over the CTAs;
//   3. every CTA reads the histogram: each key's total and the part of it in
//      earlier CTAs; one pair of block scans gives each key's first position
//      and the work list offsets;
//   4. stable scatter of this CTA's tokens into perm (a warp's first batch of
//      indices is still in registers); CTA 0 writes the slot offsets and
//      header, the work items are shared out by key.
__global__ void __launch_bounds__(kGroupThreads, 1)
group_kernel(int T, int S, const int32_t* __restrict__ idx, char* __restrict__ meta, int early) {
  extern __shared__ int smem[];
  const int K = S + 1;
  int* cnt = smem;                          // [key][kCntPitch]
  int* tot = cnt + K * kCntPitch;           // this CTA's count, then the total, per key
  int* base = tot + K;                      // first position per key
  int* pre = base + K;                      // tokens of the key in earlier CTAs
  int* ni = pre + K;                        // items per key, then item offsets
  int* scratch = ni + K;                    // 128 ints of scan scratch, 2 totals, a flag

  // the previous kernel's writes (idx, meta) are visible after this wait; with
  // `early` the indices are known not to be among them, and the wait comes
  // after counting and after the CTAs have exchanged their counts (through
  // the histogram rows and barrier words that only this kernel uses), before
  // the first write to the grouping (a kernel before this one may still read
  // the grouping held there)
  if (!early) ptx::grid_dep_wait();
  MetaLayout L(T, S);
  MetaHeader* hdr = reinterpret_cast<MetaHeader*>(meta);
  int* slot_off = reinterpret_cast<int*>(meta + L.off_slot);
  int* perm = reinterpret_cast<int*>(meta + L.off_perm);
  int4* items = reinterpret_cast<int4*>(meta + L.off_items);
  int* hist = reinterpret_cast<int*>(meta + L.off_hist);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nb = gridDim.x, cta = blockIdx.x;
  const int chunk = (T + nb - 1) / nb;
  const int c0 = min(T, cta * chunk), c1 = min(T, c0 + chunk);
  const int wchunk = (((c1 - c0) + kGroupWarps - 1) / kGroupWarps + 31) & ~31;
  const int beg = min(c1, c0 + warp * wchunk);
  const int end = min(c1, beg + wchunk);

  for (int i = tid; i < K * kCntPitch; i += kGroupThreads) cnt[i] = 0;
  __syncthreads();

  // a warp's first batch of indices stays in registers for the scatter pass
  // (the only batch while a warp's part is at most 32 * kLoadBatch tokens)
  int v0[kLoadBatch];
  int bad = 0;
  for (int b0 = beg; b0 < end; b0 += 32 * kLoadBatch) {
    int v[kLoadBatch];
#pragma unroll
    for (int u = 0; u < kLoadBatch; ++u) {
      const int t = b0 + 32 * u + lane;
      v[u] = t < end ? __ldg(idx + t) : -1;
    }
    if (b0 == beg) {
#pragma unroll
      for (int u = 0; u < kLoadBatch; ++u) v0[u] = v[u];
    }
#pragma unroll
    for (int u = 0; u < kLoadBatch; ++u) {
      if (b0 + 32 * u >= end) break;              // warp-uniform
      const int t = b0 + 32 * u + lane;
      const bool valid = t < end;
      if (valid && (v[u] < -1 || v[u] >= S)) ++bad;
      const int key = valid ? ((v[u] >= 0 && v[u] < S) ? v[u] : S) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      if (valid && lane == __ffs(peers) - 1) cnt[key * kCntPitch + warp] += __popc(peers);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if (lane == 0 && bad) atomicAdd(&hdr->bad_index, bad);
  __syncthreads();

  // key k, lane = warp w: the warp's offset among the CTA's tokens of key k,
  // and the CTA's total of key k
  for (int k = warp; k < K; k += kGroupWarps) {
    const int c = cnt[k * kCntPitch + lane];
    int inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += u;
    }
    cnt[k * kCntPitch + lane] = inc - c;
    if (lane == 31) {
      tot[k] = inc;
      if (nb > 1) hist[cta * K + k] = inc;
    }
  }
  if (nb > 1) __threadfence();
  __syncthreads();
  if (nb > 1) {
    if (tid == 0) scratch[130] = group_barrier(hdr, nb) ? 1 : 0;
    __syncthreads();
    if (!scratch[130]) {                          // another CTA never arrived
      if (tid == 0) atomicAdd(&hdr->bad_meta, 1);
      return;
    }
  }

  for (int k = tid; k < K; k += kGroupThreads) {
    int all = 0, before = 0;
    for (int c = 0; c < nb; ++c) {
      const int v = c == cta ? tot[k] : __ldcg(hist + c * K + k);
      all += v;
      before += c < cta ? v : 0;
    }
    tot[k] = all;
    base[k] = all;
    pre[k] = before;
    ni[k] = (all + kItemTokens - 1) / kItemTokens;
  }
  __syncthreads();
  // K <= LORA_MAX_SLOTS + 1 <= 2 * kGroupThreads
  block_exclusive_scan2(base, ni, K, scratch, scratch + 128, scratch + 129);
  const int n_items = scratch[129];

  // per-(key, warp) start positions
  for (int e = tid; e < K * kGroupWarps; e += kGroupThreads) {
    const int k = e / kGroupWarps, w = e % kGroupWarps;
    cnt[k * kCntPitch + w] += base[k] + pre[k];
  }
  // The next kernel may start now: this CTA no longer reads the histogram
  // rows or the barrier words, which a following grouping launch (with
  // `early`) may use before its own wait.
  __syncthreads();
  ptx::grid_dep_launch_dependents();
  if (early) ptx::grid_dep_wait();
  for (int k = tid; k < K; k += kGroupThreads) {
    if (cta == 0) slot_off[k] = base[k];
    if (k % nb == cta) {
      const int it0 = ni[k], n = tot[k];
      for (int j = 0; j * kItemTokens < n; ++j) {
        const int b0 = base[k] + j * kItemTokens;
        const int e0 = min(base[k] + n, b0 + kItemTokens);
        items[it0 + j] = make_int4(k < S ? k : -1, b0, e0, 0);
      }
    }
  }
  if (cta == 0 && tid == 0) {
    slot_off[K] = T;
    hdr->n_items = n_items;
    hdr->n_active = base[S];
    hdr->T = T;
    hdr->S = S;
  }
  __syncthreads();

  // Stable scatter: the same walk; a token's rank among equal keys of its
  // 32-token step comes from the match mask.
  for (int b0 = beg; b0 < end; b0 += 32 * kLoadBatch) {
    int v[kLoadBatch];
#pragma unroll
    for (int u = 0; u < kLoadBatch; ++u) {
      const int t = b0 + 32 * u + lane;
      v[u] = b0 == beg ? v0[u] : (t < end ? __ldg(idx + t) : -1);
    }
#pragma unroll
    for (int u = 0; u < kLoadBatch; ++u) {
      if (b0 + 32 * u >= end) break;
      const int t = b0 + 32 * u + lane;
      const bool valid = t < end;
      const int key = valid ? ((v[u] >= 0 && v[u] < S) ? v[u] : S) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      int pos = 0;
      if (valid) pos = cnt[key * kCntPitch + warp] + __popc(peers & lanemask_lt());
      __syncwarp();
      if (valid) {
        perm[pos] = t;
        if (lane == __ffs(peers) - 1) cnt[key * kCntPitch + warp] += __popc(peers);
      }
      __syncwarp();
    }
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
  ptx::grid_dep_wait();
  ptx::grid_dep_launch_dependents();
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

// Per-slot ranks into the workspace (ranks == null clears them).
__global__ void set_ranks_kernel(int S, const int32_t* __restrict__ ranks, char* __restrict__ meta) {
  MetaHeader* hdr = reinterpret_cast<MetaHeader*>(meta);
  int* dst = reinterpret_cast<int*>(meta + MetaLayout::a256(256) +
                                    MetaLayout::a256(sizeof(int) * (size_t)(S + 2)));
  if (ranks != nullptr)
    for (int g = threadIdx.x; g < S; g += blockDim.x) dst[g] = ranks[g];
  if (threadIdx.x == 0) hdr->has_ranks = ranks != nullptr ? 1 : 0;
}

}  // namespace

cudaError_t launch_set_ranks(int S, const int32_t* ranks, void* meta, cudaStream_t st) {
  set_ranks_kernel<<<1, 256, 0, st>>>(S, ranks, static_cast<char*>(meta));
  return counted_launch(cudaGetLastError());
}

size_t group_smem_bytes(int S) {
  return sizeof(int) * ((size_t)(kCntPitch + 4) * (S + 1) + 131);
}

cudaError_t launch_group(int T, int S, const int32_t* idx, void* meta, cudaStream_t st,
                         int early) {
  size_t smem = group_smem_bytes(S);
  cudaError_t e = cudaFuncSetAttribute(group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(group_ctas(T), 1, 1);
  cfg.blockDim = dim3(kGroupThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return counted_launch(
      cudaLaunchKernelEx(&cfg, group_kernel, T, S, idx, static_cast<char*>(meta), early));
}

cudaError_t launch_segment_items(int T, int S, int n_seg, const int32_t* seg_starts,
                                 const int32_t* seg_adapter, void* meta, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(kGroupThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return counted_launch(cudaLaunchKernelEx(&cfg, segment_items_kernel, T, S, n_seg, seg_starts,
                                           seg_adapter, static_cast<char*>(meta)));
}

}  // namespace lora
