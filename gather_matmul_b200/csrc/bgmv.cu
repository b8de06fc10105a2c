// CUDA-core shrink and expand over a work list of (slot, <= 16 tokens) items.
//
// These are the per-token (BGMV) kernels of "Add multi-LoRA support"
// (vllm-project/vllm pull 1804, Features list: BGMV kernels), re-designed for
// sm_100a: the tokens of a batch are first grouped by adapter slot on the
// device (group.cu), so one CTA loads an adapter tile ONCE and applies it to
// every token of its item, instead of gathering a per-token copy of the
// adapter (the copies that made the PyTorch gather baseline slow in
// "[Hardware][TPU][V1] Better tpu multilora compilation").
//
// Shrink  buf[i][t][j] = sum_d x[t][d] A_i[g][j][d]
//   A CTA of 4 warps owns (item, rank group of 8, one D-chunk).  Each lane
//   holds an 8-column slice of the 8 adapter rows in registers (fp32), reads
//   each token's 8 x values with one 128-bit load, and forms 8 partial dot
//   products.  A transposing butterfly reduces the 8 values across the 32
//   lanes with 9 shuffles; warps add their partials in shared memory; the
//   D-chunks of one item form a thread-block cluster and are summed in fixed
//   rank order through distributed shared memory.  Every sum has a fixed
//   order, so results are bitwise reproducible, and no atomics or pre-zeroed
//   output are needed.
// Expand  y[t][off_i + o] = rn(y + scale * sum_j buf_i[t][j] B_i[g][o][j])
//   A CTA of 128 threads owns (item, 128*CPL output columns of one slice).
//   Each thread keeps its CPL rows of B (CPL x r values) in registers, reads
//   the item's fp32 buf rows from shared memory (broadcast) and does a
//   coalesced read-modify-write of its CPL columns of every token's y row.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace lora {

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kJR = 8;                    // ranks per shrink CTA
constexpr int kColsPerPass = kWarps * 32 * 8;
constexpr int kPersistentCtas = 148 * 4;

// Transposing butterfly: N values per lane, summed over the 32 lanes.  After
// the call v[0] of lane l holds the total for value index jj(l); lanes with
// (l & (32/N - 1)) == 0 are the designated writers.
template <int N, int O>
struct Butterfly {
  static __device__ __forceinline__ void run(float* v, int lane, int& jj) {
    const bool up = (lane & O) != 0;
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
      float send = up ? v[k] : v[k + N / 2];
      float keep = up ? v[k + N / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, O);
    }
    if (up) jj += N / 2;
    Butterfly<N / 2, O / 2>::run(v, lane, jj);
  }
};
template <int O>
struct Butterfly<1, O> {
  static __device__ __forceinline__ void run(float* v, int, int&) {
    float s = v[0];
#pragma unroll
    for (int o = O; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    v[0] = s;
  }
};

template <typename E>
__global__ void __launch_bounds__(kThreads)
shrink_items_kernel(const ShrinkArgs a) {
  __shared__ float sacc[kWarps][kItemTokens][kJR];
  __shared__ float cpart[kItemTokens * kJR];
  __shared__ int stok[kItemTokens];

  ptx::grid_dep_wait();               // the grouping / buf producers have finished
  ptx::grid_dep_launch_dependents();
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int T = a.T, D = a.D, r = a.r;
  MetaLayout L(T, a.S);
  const int n_items = checked_items(a.meta, T, a.S);
  const int* perm = reinterpret_cast<const int*>(a.meta + L.off_perm);
  const int4* items = reinterpret_cast<const int4*>(a.meta + L.off_items);

  const int groups = r / kJR;
  const int slice = blockIdx.y / groups;
  const int j0 = (blockIdx.y % groups) * kJR;
  float* bufs = a.buf + (size_t)slice * T * r;
  const E* x = static_cast<const E*>(a.x);

  // this CTA's columns [c0, c1)
  const int Dc = ((D + CL * 8 - 1) / (CL * 8)) * 8;
  const int c0 = crank * Dc;
  const int c1 = min(D, c0 + Dc);

  const int n_clusters = gridDim.x / CL;
  for (int item = blockIdx.x / CL; item < n_items; item += n_clusters) {
    const int4 it = items[item];
    const int slot = it.x, nt = it.z - it.y;
    __syncthreads();   // previous item's readers of stok / cpart are done
    if (tid < nt) {
      // a token of a per-token grouping whose index disagrees with its group
      // (stale workspace) is skipped (-1) and counted once per item
      int tok = (it.w & kItemDirect) ? it.y + tid : perm[it.y + tid];
      if (!(it.w & kItemDirect) && !grouped_row_ok(a.idx, tok, slot, a.S)) {
        if (crank == 0 && blockIdx.y == 0) count_bad_meta(a.meta, 1);
        tok = -1;
      }
      stok[tid] = tok;
    }
    for (int e = tid; e < kWarps * kItemTokens * kJR; e += kThreads)
      (&sacc[0][0][0])[e] = 0.f;
    __syncthreads();

    // tokens without an adapter, and rank groups past the slot's own rank:
    // zero buf columns, nothing read
    if (slot < 0 || j0 >= slot_rank(a.meta, a.S, slot, r)) {
      if (crank == 0)
        for (int e = tid; e < nt * kJR; e += kThreads)
          if (stok[e / kJR] >= 0) bufs[(size_t)stok[e / kJR] * r + j0 + e % kJR] = 0.f;
      continue;
    }

    const E* Ag = static_cast<const E*>(a.A[slice]) + ((size_t)slot * r + j0) * D;
    for (int col0 = c0 + warp * 256; col0 < c1; col0 += kColsPerPass) {
      const int col = col0 + lane * 8;
      const bool inb = col < c1;
      float av[kJR][8];
#pragma unroll
      for (int j = 0; j < kJR; ++j) {
        uint4 u = inb ? ldg_stream(Ag + (size_t)j * D + col) : make_uint4(0, 0, 0, 0);
        Elem<E>::to_f32(u, av[j]);
      }
      for (int k0 = 0; k0 < nt; k0 += 4) {
        uint4 xu[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = k0 + q;
          xu[q] = (inb && k < nt && stok[k] >= 0) ? ldg_nc(x + (size_t)stok[k] * a.ldx + col)
                                                  : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = k0 + q;
          if (k >= nt) break;
          float xf[8];
          Elem<E>::to_f32(xu[q], xf);
          float p[kJR];
#pragma unroll
          for (int j = 0; j < kJR; ++j) {
            float s = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) s = fmaf(av[j][u], xf[u], s);
            p[j] = s;
          }
          int jj = 0;
          Butterfly<kJR, 16>::run(p, lane, jj);
          if ((lane & (32 / kJR - 1)) == 0) sacc[warp][k][jj] += p[0];
        }
      }
    }
    __syncthreads();
    for (int e = tid; e < nt * kJR; e += kThreads) {
      const int k = e / kJR, j = e % kJR;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += sacc[w][k][j];
      cpart[e] = s;
    }
    if (CL == 1) {
      __syncthreads();
      for (int e = tid; e < nt * kJR; e += kThreads)
        if (stok[e / kJR] >= 0) bufs[(size_t)stok[e / kJR] * r + j0 + e % kJR] = cpart[e];
    } else {
      cluster.sync();      // every CTA's cpart is complete
      const int per = (nt * kJR + CL - 1) / CL;
      const int e0 = crank * per, e1 = min(nt * kJR, e0 + per);
      for (int e = e0 + tid; e < e1; e += kThreads) {
        float s = 0.f;
        for (int q = 0; q < CL; ++q) s += cluster.map_shared_rank(cpart, q)[e];
        if (stok[e / kJR] >= 0) bufs[(size_t)stok[e / kJR] * r + j0 + e % kJR] = s;
      }
      cluster.sync();      // no CTA reuses cpart while a peer still reads it
    }
  }
}

template <int CPL> struct YVec;
template <> struct YVec<2> {
  using T = uint32_t;
  static __device__ __forceinline__ T load(const void* p) { return *static_cast<const uint32_t*>(p); }
};
template <> struct YVec<4> {
  using T = uint2;
  static __device__ __forceinline__ T load(const void* p) { return *static_cast<const uint2*>(p); }
};
template <> struct YVec<8> {
  using T = uint4;
  static __device__ __forceinline__ T load(const void* p) { return *static_cast<const uint4*>(p); }
};

template <typename E, int R, int CPL>
__global__ void __launch_bounds__(kThreads)
expand_items_kernel(const ExpandArgs a) {
  __shared__ __align__(16) float sbuf[kItemTokens][R];
  __shared__ int stok[kItemTokens];
  using YV = YVec<CPL>;
  constexpr int OC = kThreads * CPL;

  ptx::grid_dep_wait();
  ptx::grid_dep_launch_dependents();
  const int tid = threadIdx.x;
  MetaLayout L(a.T, a.S);
  const int n_items = checked_items(a.meta, a.T, a.S);
  const int* perm = reinterpret_cast<const int*>(a.meta + L.off_perm);
  const int4* items = reinterpret_cast<const int4*>(a.meta + L.off_items);
  const int total_chunks = a.chunk_base[a.n_slices];
  const long units = (long)n_items * total_chunks;

  for (long w = blockIdx.x; w < units; w += gridDim.x) {
    const int item = (int)(w / total_chunks);
    const int ch = (int)(w % total_chunks);
    const int4 it = items[item];
    const int slot = it.x, nt = it.z - it.y;
    if (slot < 0) continue;    // uniform across the CTA
    int slice = 0;
#pragma unroll 1
    while (ch >= a.chunk_base[slice + 1]) ++slice;
    const int o0 = (ch - a.chunk_base[slice]) * OC + tid * CPL;
    const bool active = o0 < a.D_out[slice];
    const float* bsl = a.buf + (size_t)slice * a.buf_slice_stride;

    __syncthreads();   // previous unit's readers of sbuf / stok are done
    if (tid < nt) {
      // tokens whose index disagrees with their group (stale workspace) are
      // neither read nor written; counted once per item
      int tok = (it.w & kItemDirect) ? it.y + tid : perm[it.y + tid];
      if (!(it.w & kItemDirect) && !grouped_row_ok(a.idx, tok, slot, a.S)) {
        if (ch == 0) count_bad_meta(a.meta, 1);
        tok = -1;
      }
      stok[tid] = tok;
    }
    __syncthreads();
    for (int e = tid; e < nt * R; e += kThreads)
      sbuf[e / R][e % R] = stok[e / R] >= 0 ? bsl[(size_t)stok[e / R] * R + e % R] : 0.f;
    __syncthreads();
    if (!active) continue;

    // this thread's CPL rows of B_i[slot], the slot's own rank k of its r
    // values each (the padding past k is neither read nor multiplied), as fp32
    const int kslot = slot_rank(a.meta, a.S, slot, R);
    float bf[CPL][R];
    const E* Bg = static_cast<const E*>(a.B[slice]) + ((size_t)slot * a.D_out[slice] + o0) * R;
#pragma unroll
    for (int c = 0; c < CPL; ++c)
#pragma unroll
      for (int j8 = 0; j8 < R / 8; ++j8) {
        uint4 u = j8 * 8 < kslot ? ldg_stream(Bg + c * R + j8 * 8) : make_uint4(0, 0, 0, 0);
        Elem<E>::to_f32(u, &bf[c][j8 * 8]);
      }

    E* ybase = static_cast<E*>(a.y) + a.y_col_off[slice] + o0;
    for (int k0 = 0; k0 < nt; k0 += 8) {
      typename YV::T yv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (k0 + q < nt && stok[k0 + q] >= 0) yv[q] = YV::load(ybase + (size_t)stok[k0 + q] * a.ldy);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int k = k0 + q;
        if (k >= nt) break;
        if (stok[k] < 0) continue;
        float acc[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
#pragma unroll
        for (int j4 = 0; j4 < R / 4; ++j4) {
          if (j4 * 4 >= kslot) break;
          const float4 bv = *reinterpret_cast<const float4*>(&sbuf[k][j4 * 4]);
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            acc[c] = fmaf(bv.x, bf[c][j4 * 4 + 0], acc[c]);
            acc[c] = fmaf(bv.y, bf[c][j4 * 4 + 1], acc[c]);
            acc[c] = fmaf(bv.z, bf[c][j4 * 4 + 2], acc[c]);
            acc[c] = fmaf(bv.w, bf[c][j4 * 4 + 3], acc[c]);
          }
        }
        uint16_t* yh = reinterpret_cast<uint16_t*>(&yv[q]);
#pragma unroll
        for (int c = 0; c < CPL; ++c)
          yh[c] = Elem<E>::from_f32(fmaf(a.scale, acc[c], Elem<E>::to_f32(yh[c])));
        *reinterpret_cast<typename YV::T*>(ybase + (size_t)stok[k] * a.ldy) = yv[q];
      }
    }
  }
}

template <typename E>
cudaError_t shrink_dispatch(const ShrinkArgs& a, int max_items, cudaStream_t st) {
  // D-chunks per item: one pass of 1024 columns per CTA where possible, at
  // most 8 CTAs (portable cluster size).
  int CL = (a.D + kColsPerPass - 1) / kColsPerPass;
  if (CL > 8) CL = 8;
  if (CL < 1) CL = 1;
  int clusters = max_items;
  int cap = kPersistentCtas / CL;
  if (clusters > cap) clusters = cap;
  if (clusters < 1) clusters = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(clusters * CL, a.n_slices * (a.r / kJR), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return counted_launch(cudaLaunchKernelEx(&cfg, shrink_items_kernel<E>, a));
}

template <typename E, int R, int CPL>
cudaError_t expand_launch(const ExpandArgs& a, int max_items, cudaStream_t st) {
  long units = (long)max_items * a.chunk_base[a.n_slices];
  int grid = units < kPersistentCtas ? (int)units : kPersistentCtas;
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return counted_launch(cudaLaunchKernelEx(&cfg, expand_items_kernel<E, R, CPL>, a));
}

template <typename E>
cudaError_t expand_dispatch(ExpandArgs a, int max_items, cudaStream_t st) {
  int cpl = a.r == 8 ? 8 : a.r == 16 ? 4 : 2;
  int oc = kThreads * cpl;
  a.chunk_base[0] = 0;
  for (int i = 0; i < a.n_slices; ++i)
    a.chunk_base[i + 1] = a.chunk_base[i] + (a.D_out[i] + oc - 1) / oc;
  switch (a.r) {
    case 8: return expand_launch<E, 8, 8>(a, max_items, st);
    case 16: return expand_launch<E, 16, 4>(a, max_items, st);
    case 32: return expand_launch<E, 32, 2>(a, max_items, st);
    case 64: return expand_launch<E, 64, 2>(a, max_items, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_shrink_items(lora_dtype dt, const ShrinkArgs& a, int max_items,
                                cudaStream_t st) {
  return dt == LORA_BF16 ? shrink_dispatch<__nv_bfloat16>(a, max_items, st)
                         : shrink_dispatch<__half>(a, max_items, st);
}

cudaError_t launch_expand_items(lora_dtype dt, ExpandArgs a, int max_items, cudaStream_t st) {
  return dt == LORA_BF16 ? expand_dispatch<__nv_bfloat16>(a, max_items, st)
                         : expand_dispatch<__half>(a, max_items, st);
}

}  // namespace lora
