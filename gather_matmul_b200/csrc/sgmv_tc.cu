// Segment-grouped (SGMV) shrink and expand on the 5th-generation tensor
// cores (tcgen05), for prefill-sized segments.
//
// "Add multi-LoRA support" (vllm-project/vllm pull 1804), Limitations list:
// the per-token BGMV kernel is not efficient for prefill, and the CUTLASS SGMV
// kernel of the time lost accuracy because its intermediate was stored in half
// precision.  Here a segment of tokens sharing one adapter is a dense
// contraction and runs on tcgen05 tensor cores, while the intermediate stays
// fp32 end to end:
//
// Shrink  buf[rows][:] = X[rows][:] . A[a]^T     M = 128 tokens, N = r, K = D
//   One CTA per (128-row tile of a segment, K-split); a cluster of KS CTAs
//   covers the K range of one tile.  A 4-6 stage pipeline of 64-wide K blocks:
//   TMA loads the x tile (128 x 64, 128-byte swizzle) and the adapter tile
//   (r x 64); one thread issues tcgen05.mma (kind::f16, fp32 accumulator in
//   tensor memory) and tcgen05.commit frees the stage.  The accumulator is read
//   back with tcgen05.ld; split-K partials are summed in rank order through
//   distributed shared memory (deterministic, no atomics).
// Expand  Y[rows][cols] += scale * buf[rows][:] . B[a][cols]^T   M = 128, N = 128, K = r
//   One CTA per (tile, 128 output columns, slice).  The fp32 intermediate
//   enters the tensor core as hi + lo of the input type after an exact
//   power-of-two rescale per row (about 16 bits for bf16, 22 for fp16), two
//   MMAs per K step into one fp32 accumulator.  The B tile arrives by TMA;
//   each thread prefetches its row's y values into registers at the start
//   (whole 32-byte sectors), so four CTAs fit per SM; the epilogue adds
//   scale * acc with one round-to-nearest-even and stores from registers.
//   Rows past the segment are never written.
//
// Every mbarrier wait is bounded (about one second); a timeout is counted in
// the workspace and the kernel still releases its tensor memory and exits.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace lora {

namespace {

constexpr int kTM = 128;          // token rows per tile (MMA M)
constexpr int kBK = 64;           // K elements per pipeline stage: one 128-byte row
template <int R>
constexpr int stages_for() { return R <= 32 ? 6 : 4; }   // two CTAs per SM at every rank
constexpr int kThreads = 128;     // 4 warps: one per 32 TMEM lanes
constexpr int kNT = 128;          // expand output columns per CTA (MMA N)

struct TileInfo {
  int seg, m0, valid, adapter;
};

// Tile `tile` of the segment list, segments clamped into [0, T] so that no
// access can leave the buffers even for malformed lists (those are counted
// separately).  Warp-cooperative; every lane returns the same answer.
__device__ bool find_tile(int tile, const int32_t* __restrict__ ss,
                          const int32_t* __restrict__ sa, int n_seg, int T, TileInfo& ti,
                          int implicit_slots) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int s0 = 0; s0 < n_seg; s0 += 32) {
    const int s = s0 + lane;
    int a = 0, b = 0;
    if (s < n_seg) {
      a = min(max(ss[s], 0), T);
      b = max(a, min(max(ss[s + 1], 0), T));
    }
    const int nt = (b - a + kTM - 1) / kTM;
    int inc = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    const int total = __shfl_sync(0xffffffffu, inc, 31);
    if (tile < base + total) {
      const unsigned m = __ballot_sync(0xffffffffu, s < n_seg && base + inc > tile);
      const int l = __ffs(m) - 1;
      const int sa_l = __shfl_sync(0xffffffffu, a, l);
      const int sb_l = __shfl_sync(0xffffffffu, b, l);
      const int excl = __shfl_sync(0xffffffffu, inc - nt, l);
      ti.seg = s0 + l;
      ti.m0 = sa_l + (tile - base - excl) * kTM;
      ti.valid = min(kTM, sb_l - ti.m0);
      // per-token grouping: segment g is slot g, the last one holds the tokens
      // without an adapter
      ti.adapter = implicit_slots ? (s0 + l < implicit_slots ? s0 + l : -1) : sa[s0 + l];
      return true;
    }
    base += total;
  }
  return false;
}

// One CTA per launch counts malformed lists and out-of-range adapters.
__device__ void validate_segments(const int32_t* ss, const int32_t* sa, int n_seg, int T, int S,
                                  int* bad_index, int* bad_meta) {
  int bad = 0, badi = 0;
  if (threadIdx.x == 0 && (ss[0] != 0 || ss[n_seg] != T)) bad = 1;
  for (int s = threadIdx.x; s < n_seg; s += blockDim.x) {
    const int a = ss[s], b = ss[s + 1];
    if (b < a || a < 0 || b > T) bad = 1;
    const int ad = sa[s];
    if ((ad < -1 || ad >= S) && b > a) badi += b - a;
  }
  if (bad) atomicAdd(bad_meta, 1);
  if (badi) atomicAdd(bad_index, badi);
}

// The per-token grouping in the workspace was built for (T, S): otherwise its
// positions are not known to lie in this call's buffers, so nothing is done
// and the error is counted once (the error counters head the workspace).
__device__ bool grouped_meta_ok(int* counters, int T, int S) {
  const MetaHeader* h = reinterpret_cast<const MetaHeader*>(counters);
  if (h->T == T && h->S == S) return true;
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0)
    atomicAdd(&reinterpret_cast<MetaHeader*>(counters)->bad_meta, 1);
  return false;
}

template <int SW>
__device__ __forceinline__ int swz(int row, int chunk) {
  if constexpr (SW == 128) return chunk ^ (row & 7);
  else if constexpr (SW == 64) return chunk ^ ((row >> 1) & 3);
  else return chunk ^ ((row >> 2) & 1);
}

struct ShrinkTCParams {
  CUtensorMap tmX;                       // x as [T rows, D cols], box {64, 128} (or {64, 1}
                                         // for row gathers), 128B swizzle
  CUtensorMap tmA[LORA_MAX_SLICES];      // A_i as [S*r rows, D cols], box {64, r}, 128B swizzle
  const int32_t* seg_starts;
  const int32_t* seg_adapter;
  int n_seg;
  float* buf;
  const int32_t* perm;                   // row p of a tile is token perm[p]; null = identity
  int implicit_slots;                    // > 0: segment g is slot g (per-token grouping)
  int T, D, S, n_slices, KS;
  int* bad_index;
  int* bad_meta;
};

template <int R>
struct ShrinkSmem {
  static constexpr int kXBytes = kTM * 128;
  static constexpr int kABytes = R * 128;
  static constexpr int kStageBytes = kXBytes + kABytes;   // multiple of 1024
  static constexpr int kPitch = R + 4;                     // floats, partial-sum rows
  static constexpr int kStages = stages_for<R>();
  static constexpr size_t kBar = (size_t)kStageBytes * kStages;
  static constexpr size_t kTotal = kBar + 8 * (2 * kStages + 1) + 64 + 1024;
};

template <typename E, int R>
__global__ void __launch_bounds__(kThreads, 2)
sgmv_shrink_tc_kernel(const __grid_constant__ ShrinkTCParams P) {
  using L = ShrinkSmem<R>;
  constexpr int kStages = L::kStages;
  constexpr bool kBF = std::is_same<E, __nv_bfloat16>::value;
  constexpr uint32_t kIdesc = ptx::umma_idesc_f16(kBF, kTM, R);
  constexpr uint32_t kTmemCols = R < 32 ? 32 : R;
  cg::cluster_group cluster = cg::this_cluster();
  const int KS = P.KS;
  const int kr = (int)cluster.block_rank();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.y;

  extern __shared__ char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + kStages;
  uint64_t* accbar = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accbar + 1);
  int* sinfo = reinterpret_cast<int*>(tmem_slot + 4);

  if (blockIdx.x == 0 && slice == 0 && !P.implicit_slots)
    validate_segments(P.seg_starts, P.seg_adapter, P.n_seg, P.T, P.S, P.bad_index, P.bad_meta);
  // grouping metadata must have been built for this call's sizes
  const bool meta_ok = !P.implicit_slots || grouped_meta_ok(P.bad_index, P.T, P.S);
  if (warp == 0) {
    TileInfo ti;
    const bool found = meta_ok && find_tile(blockIdx.x / KS, P.seg_starts, P.seg_adapter,
                                            P.n_seg, P.T, ti, P.implicit_slots);
    if (lane == 0) {
      sinfo[0] = found ? 1 : 0;
      sinfo[1] = ti.m0;
      sinfo[2] = ti.valid;
      sinfo[3] = ti.adapter;
    }
  }
  __syncthreads();
  if (!sinfo[0]) return;                      // same for the whole cluster
  const int m0 = sinfo[1], valid = sinfo[2], adapter = sinfo[3];
  float* bufs = P.buf + (size_t)slice * P.T * R;
  const int32_t* perm = P.perm;
  auto token = [&](int p) { return perm ? perm[p] : p; };
  if (adapter < 0 || adapter >= P.S) {        // no adapter: zero rows (rank 0 writes them)
    if (kr == 0)
      for (int e = tid; e < valid * R; e += kThreads) bufs[(size_t)token(m0 + e / R) * R + e % R] = 0.f;
    return;
  }

  const int nkb_all = (P.D + kBK - 1) / kBK;
  const int kb0 = kr * nkb_all / KS, kb1 = (kr + 1) * nkb_all / KS;
  const int nkb = kb1 - kb0;                  // >= 1 (the host keeps KS <= nkb_all)

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accbar, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&P.tmX);
    ptx::prefetch_tensormap(&P.tmA[slice]);
  }
  if (warp == 0) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  const int ngroups = (valid + 3) / 4;        // 4-row gathers per stage (row indirection)
  const uint32_t stage_bytes =
      perm ? (uint32_t)(ngroups * 4 * 128 + L::kABytes) : (uint32_t)L::kStageBytes;
  if (warp == 0) {
    // producer warp: x tile (one 2-D tile, or up to 32 row gathers issued by
    // the 32 lanes) and the adapter tile into stage s
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      if (i >= kStages) ok &= ptx::mbar_wait(&empty[s], ph ^ 1);   // MMAs of i - kStages done
      char* st = smem + (size_t)s * L::kStageBytes;
      const int kx = (kb0 + i) * kBK;
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(&full[s], stage_bytes);
        ptx::tma_load_2d(st + L::kXBytes, &P.tmA[slice], kx, adapter * R, &full[s]);
        if (!perm) ptx::tma_load_2d(st, &P.tmX, kx, m0, &full[s]);
      }
      __syncwarp();
      if (perm && lane < ngroups) {
        int rr[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int p = m0 + 4 * lane + j;
          rr[j] = perm[p < m0 + valid ? p : m0];
        }
        ptx::tma_gather4(st + lane * 4 * 128, &P.tmX, kx, rr[0], rr[1], rr[2], rr[3], &full[s]);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    const uint32_t sbase = ptx::smem_u32(smem);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      ok &= ptx::mbar_wait(&full[s], ph);
      ptx::tc_fence_after();
      const uint32_t xa = sbase + s * L::kStageBytes, aa = xa + L::kXBytes;
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k)
        ptx::tc_mma_f16(tmem, ptx::umma_desc_kmajor(xa + k * 32, 128),
                        ptx::umma_desc_kmajor(aa + k * 32, 128), kIdesc, (i > 0 || k > 0) ? 1u : 0u);
      ptx::tc_commit(&empty[s]);              // stage s is free once these MMAs finish
    }
    ptx::tc_commit(accbar);
  }
  ok &= ptx::mbar_wait(accbar, 0);
  ptx::tc_fence_after();

  // accumulator row m = 32 * warp + lane, r fp32 columns
  float v[R];
#pragma unroll
  for (int c = 0; c < R / 16; ++c) {
    uint32_t r[16];
    ptx::tc_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c * 16, r);
    ptx::tc_wait_ld();
#pragma unroll
    for (int u = 0; u < 16; ++u) v[c * 16 + u] = __uint_as_float(r[u]);
  }
  const int m = warp * 32 + lane;
  if (KS == 1) {
    if (m < valid) {
      float4* row = reinterpret_cast<float4*>(bufs + (size_t)token(m0 + m) * R);
#pragma unroll
      for (int q = 0; q < R / 4; ++q) row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  } else {
    // every stage is drained (accbar): reuse the stage memory for partials
    float* part = reinterpret_cast<float*>(smem);
#pragma unroll
    for (int q = 0; q < R / 4; ++q)
      *reinterpret_cast<float4*>(part + m * L::kPitch + 4 * q) =
          make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    cluster.sync();
    const int rows = kTM / KS;                // rank kr sums rows [kr*rows, (kr+1)*rows)
    for (int e = tid; e < rows * R; e += kThreads) {
      const int mm = kr * rows + e / R, j = e % R;
      float s = 0.f;
      for (int q = 0; q < KS; ++q) s += cluster.map_shared_rank(part, q)[mm * L::kPitch + j];
      if (mm < valid) bufs[(size_t)token(m0 + mm) * R + j] = s;
    }
    cluster.sync();                           // peers are done reading this CTA's partials
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
  if (!ok && tid == 0) atomicAdd(P.bad_meta, 1);
}

struct ExpandTCParams {
  CUtensorMap tmB[LORA_MAX_SLICES];      // B_i as [S*D_out_i rows, r cols], box {r, 128}
  const float* buf;
  int64_t buf_slice_stride;
  void* y;
  int64_t ldy;
  int64_t y_col_off[LORA_MAX_SLICES];
  int D_out[LORA_MAX_SLICES];
  const int32_t* seg_starts;
  const int32_t* seg_adapter;
  int n_seg;
  const int32_t* perm;                   // row p of a tile is token perm[p]; null = identity
  int implicit_slots;                    // > 0: segment g is slot g (per-token grouping)
  int T, S, n_slices;
  float scale;
  int* bad_index;
  int* bad_meta;
};

template <int R>
struct ExpandSmem {
  static constexpr int kRowBytes = R * 2;                 // = swizzle width
  static constexpr int kBBytes = kNT * kRowBytes;
  static constexpr int kHBytes = kTM * kRowBytes;
  static constexpr size_t kOffB = 0, kOffHi = kBBytes, kOffLo = kOffHi + kHBytes,
                          kOffBar = kOffLo + kHBytes;
  static constexpr size_t kTotal = kOffBar + 8 * 2 + 64 + 1024;
};

template <typename E, int R>
__global__ void __launch_bounds__(kThreads, 4)
sgmv_expand_tc_kernel(const __grid_constant__ ExpandTCParams P) {
  using L = ExpandSmem<R>;
  constexpr bool kBF = std::is_same<E, __nv_bfloat16>::value;
  constexpr uint32_t kIdesc = ptx::umma_idesc_f16(kBF, kTM, kNT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.z;
  const int Dout = P.D_out[slice];
  const int n0 = blockIdx.y * kNT;
  if (n0 >= Dout) return;
  const int nn = min(kNT, Dout - n0);

  extern __shared__ char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  char* sB = smem + L::kOffB;
  char* sHi = smem + L::kOffHi;
  char* sLo = smem + L::kOffLo;
  uint64_t* barB = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* accbar = barB + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barB + 2);
  int* sinfo = reinterpret_cast<int*>(tmem_slot + 4);

  if (blockIdx.x == 0 && blockIdx.y == 0 && slice == 0 && !P.implicit_slots)
    validate_segments(P.seg_starts, P.seg_adapter, P.n_seg, P.T, P.S, P.bad_index, P.bad_meta);
  const bool meta_ok = !P.implicit_slots || grouped_meta_ok(P.bad_index, P.T, P.S);
  if (warp == 0) {
    TileInfo ti;
    const bool found = meta_ok && find_tile(blockIdx.x, P.seg_starts, P.seg_adapter, P.n_seg,
                                            P.T, ti, P.implicit_slots);
    if (lane == 0) {
      sinfo[0] = found && ti.adapter >= 0 && ti.adapter < P.S ? 1 : 0;
      sinfo[1] = ti.m0;
      sinfo[2] = ti.valid;
      sinfo[3] = ti.adapter;
    }
  }
  __syncthreads();
  if (!sinfo[0]) return;                 // no tile, or rows without an adapter: untouched
  const int m0 = sinfo[1], valid = sinfo[2], adapter = sinfo[3];
  E* y = static_cast<E*>(P.y) + P.y_col_off[slice] + n0;

  if (tid == 0) {
    ptx::mbar_init(barB, 1);
    ptx::mbar_init(accbar, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&P.tmB[slice]);
  }
  if (warp == 0) {
    ptx::tmem_alloc(tmem_slot, kNT);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // B tile (rows adapter*Dout + n0 ..) by TMA
  if (tid == 0) {
    ptx::mbar_arrive_expect_tx(barB, L::kBBytes);
    ptx::tma_load_2d(sB, &P.tmB[slice], 0, adapter * Dout + n0, barB);
  }
  // this thread's row of y, prefetched into registers (one 32-byte sector per
  // 16 columns) while the tile's operands are prepared
  const int m = tid;
  const int tok = m < valid ? (P.perm ? P.perm[m0 + m] : m0 + m) : 0;
  E* yrow = y + (size_t)tok * P.ldy;
  uint4 yv[kNT / 8];
#pragma unroll
  for (int c = 0; c < kNT / 8; ++c)
    yv[c] = (m < valid && c * 8 < nn) ? *reinterpret_cast<const uint4*>(yrow + c * 8)
                                      : make_uint4(0, 0, 0, 0);

  // row m's intermediate -> hi / lo operand rows (swizzled K-major), with an
  // exact power-of-two rescale 2^(7-e), e the exponent of max |buf| of the row
  float inv = 1.f;
  {
    const float4* brow = reinterpret_cast<const float4*>(
        P.buf + (size_t)slice * P.buf_slice_stride + (size_t)tok * R);
    float mx = 0.f;                        // pass 1: the row's max |value|
#pragma unroll
    for (int q = 0; q < R / 4; ++q) {
      const float4 f = m < valid ? brow[q] : make_float4(0.f, 0.f, 0.f, 0.f);
      mx = fmaxf(fmaxf(fmaxf(mx, fabsf(f.x)), fmaxf(fabsf(f.y), fabsf(f.z))), fabsf(f.w));
    }
    int e = ((__float_as_int(mx) >> 23) & 0xff) - 127;
    e = (mx > 0.f && e > -100 && e < 100) ? e : 0;
    const float sc = __int_as_float((127 - e + 7) << 23);
    inv = __int_as_float((127 + e - 7) << 23);
#pragma unroll
    for (int c = 0; c < R / 8; ++c) {      // pass 2 (L1 hits): 8 values at a time
      float4 f0 = make_float4(0.f, 0.f, 0.f, 0.f), f1 = f0;
      if (m < valid) {
        f0 = brow[2 * c];
        f1 = brow[2 * c + 1];
      }
      const float x8[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
      uint16_t hi[8], lo[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float x = x8[u] * sc;
        hi[u] = Elem<E>::from_f32(x);
        lo[u] = Elem<E>::from_f32(x - Elem<E>::to_f32(hi[u]));
      }
      const int off = m * L::kRowBytes + swz<L::kRowBytes>(m, c) * 16;
      *reinterpret_cast<uint4*>(sHi + off) = *reinterpret_cast<const uint4*>(hi);
      *reinterpret_cast<uint4*>(sLo + off) = *reinterpret_cast<const uint4*>(lo);
    }
  }
  ptx::fence_proxy_async_smem();           // generic writes -> tensor-core operand reads
  __syncthreads();

  bool ok = true;
  if (tid == 0) {
    ok &= ptx::mbar_wait(barB, 0);
    ptx::tc_fence_after();
    const uint32_t hb = ptx::smem_u32(sHi), lb = ptx::smem_u32(sLo), bb = ptx::smem_u32(sB);
#pragma unroll
    for (int ks = 0; ks < R / 16; ++ks)
      ptx::tc_mma_f16(tmem, ptx::umma_desc_kmajor(hb + ks * 32, L::kRowBytes),
                      ptx::umma_desc_kmajor(bb + ks * 32, L::kRowBytes), kIdesc, ks > 0 ? 1u : 0u);
#pragma unroll
    for (int ks = 0; ks < R / 16; ++ks)
      ptx::tc_mma_f16(tmem, ptx::umma_desc_kmajor(lb + ks * 32, L::kRowBytes),
                      ptx::umma_desc_kmajor(bb + ks * 32, L::kRowBytes), kIdesc, 1u);
    ptx::tc_commit(accbar);
  }
  ok &= ptx::mbar_wait(accbar, 0);
  ptx::tc_fence_after();

  // epilogue: TMEM lane m = this thread's row; 16 columns at a time, one
  // fp32 fma and one rounding per element, stores straight from registers
  for (int c = 0; c < kNT / 16; ++c) {
    uint32_t r[16];
    ptx::tc_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c * 16, r);
    ptx::tc_wait_ld();
    if (m < valid && c * 16 < nn) {
      uint16_t* h = reinterpret_cast<uint16_t*>(&yv[2 * c]);
#pragma unroll
      for (int u = 0; u < 16; ++u)
        h[u] = Elem<E>::from_f32(fmaf(P.scale, __uint_as_float(r[u]) * inv, Elem<E>::to_f32(h[u])));
      reinterpret_cast<uint4*>(yrow + c * 16)[0] = yv[2 * c];
      if (c * 16 + 8 < nn) reinterpret_cast<uint4*>(yrow + c * 16)[1] = yv[2 * c + 1];
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, kNT);
  if (!ok && tid == 0) atomicAdd(P.bad_meta, 1);
}

template <typename E, int R>
cudaError_t shrink_tc_launch(const ShrinkArgs& a, const SegArgs& sg, lora_dtype dt,
                             cudaStream_t st, const int32_t* perm, int implicit_slots) {
  ShrinkTCParams P;
  memset(&P, 0, sizeof(P));
  // row gathers need a box one row high
  cudaError_t e = encode_tmap_2d(&P.tmX, dt, a.x, (uint64_t)a.D, (uint64_t)a.T,
                                 (uint64_t)a.ldx * 2, kBK, perm ? 1 : kTM, 128);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < a.n_slices; ++i) {
    e = encode_tmap_2d(&P.tmA[i], dt, a.A[i], (uint64_t)a.D, (uint64_t)a.S * R,
                       (uint64_t)a.D * 2, kBK, R, 128);
    if (e != cudaSuccess) return e;
  }
  const MetaHeader* hdr = reinterpret_cast<const MetaHeader*>(a.meta);
  P.seg_starts = sg.seg_starts;
  P.seg_adapter = sg.seg_adapter;
  P.n_seg = sg.n_seg;
  P.buf = a.buf;
  P.perm = perm;
  P.implicit_slots = implicit_slots;
  P.T = a.T;
  P.D = a.D;
  P.S = a.S;
  P.n_slices = a.n_slices;
  P.bad_index = const_cast<int*>(&hdr->bad_index);
  P.bad_meta = const_cast<int*>(&hdr->bad_meta);
  const int max_tiles = (a.T + kTM - 1) / kTM + sg.n_seg;
  const int nkb_all = (a.D + kBK - 1) / kBK;
  // split K across a cluster when there are too few tiles to fill the GPU
  int KS = 1;
  while (KS < 4 && (long)max_tiles * a.n_slices * KS < 148 && nkb_all >= 4 * KS) KS *= 2;
  P.KS = KS;
  auto kern = sgmv_shrink_tc_kernel<E, R>;
  const size_t smem = ShrinkSmem<R>::kTotal;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(max_tiles * KS, a.n_slices, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

template <typename E, int R>
cudaError_t expand_tc_launch(const ExpandArgs& a, const SegArgs& sg, lora_dtype dt,
                             cudaStream_t st, const int32_t* perm, int implicit_slots) {
  ExpandTCParams P;
  memset(&P, 0, sizeof(P));
  int max_nt = 0;
  for (int i = 0; i < a.n_slices; ++i) {
    cudaError_t e = encode_tmap_2d(&P.tmB[i], dt, a.B[i], (uint64_t)R,
                                   (uint64_t)a.S * a.D_out[i], (uint64_t)R * 2, R, kNT, R * 2);
    if (e != cudaSuccess) return e;
    P.y_col_off[i] = a.y_col_off[i];
    P.D_out[i] = a.D_out[i];
    max_nt = max(max_nt, (a.D_out[i] + kNT - 1) / kNT);
  }
  const MetaHeader* hdr = reinterpret_cast<const MetaHeader*>(a.meta);
  P.buf = a.buf;
  P.buf_slice_stride = a.buf_slice_stride;
  P.y = a.y;
  P.ldy = a.ldy;
  P.seg_starts = sg.seg_starts;
  P.seg_adapter = sg.seg_adapter;
  P.n_seg = sg.n_seg;
  P.perm = perm;
  P.implicit_slots = implicit_slots;
  P.T = a.T;
  P.S = a.S;
  P.n_slices = a.n_slices;
  P.scale = a.scale;
  P.bad_index = const_cast<int*>(&hdr->bad_index);
  P.bad_meta = const_cast<int*>(&hdr->bad_meta);
  const int max_tiles = (a.T + kTM - 1) / kTM + sg.n_seg;
  auto kern = sgmv_expand_tc_kernel<E, R>;
  const size_t smem = ExpandSmem<R>::kTotal;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(max_tiles, max_nt, a.n_slices), kThreads, smem, st>>>(P);
  return cudaGetLastError();
}

}  // namespace

namespace {
cudaError_t shrink_tc_any(lora_dtype dt, const ShrinkArgs& a, const SegArgs& s, cudaStream_t st,
                          const int32_t* perm, int implicit) {
  if (a.D % 8 != 0 || a.ldx % 8 != 0) return cudaErrorNotSupported;
  const bool bf = dt == LORA_BF16;
  switch (a.r) {
    case 16: return bf ? shrink_tc_launch<__nv_bfloat16, 16>(a, s, dt, st, perm, implicit)
                       : shrink_tc_launch<__half, 16>(a, s, dt, st, perm, implicit);
    case 32: return bf ? shrink_tc_launch<__nv_bfloat16, 32>(a, s, dt, st, perm, implicit)
                       : shrink_tc_launch<__half, 32>(a, s, dt, st, perm, implicit);
    case 64: return bf ? shrink_tc_launch<__nv_bfloat16, 64>(a, s, dt, st, perm, implicit)
                       : shrink_tc_launch<__half, 64>(a, s, dt, st, perm, implicit);
    default: return cudaErrorNotSupported;     // rank 8: no M=128 tensor-core shape
  }
}
cudaError_t expand_tc_any(lora_dtype dt, const ExpandArgs& a, const SegArgs& s, cudaStream_t st,
                          const int32_t* perm, int implicit) {
  const bool bf = dt == LORA_BF16;
  switch (a.r) {
    case 16: return bf ? expand_tc_launch<__nv_bfloat16, 16>(a, s, dt, st, perm, implicit)
                       : expand_tc_launch<__half, 16>(a, s, dt, st, perm, implicit);
    case 32: return bf ? expand_tc_launch<__nv_bfloat16, 32>(a, s, dt, st, perm, implicit)
                       : expand_tc_launch<__half, 32>(a, s, dt, st, perm, implicit);
    case 64: return bf ? expand_tc_launch<__nv_bfloat16, 64>(a, s, dt, st, perm, implicit)
                       : expand_tc_launch<__half, 64>(a, s, dt, st, perm, implicit);
    default: return cudaErrorNotSupported;
  }
}
// The per-token grouping as a segment list over the permuted token order:
// slot g's tokens are positions [slot_off[g], slot_off[g+1]) of perm, and the
// final range [slot_off[S], T) holds the tokens without an adapter.
SegArgs grouped_segments(const char* meta, int T, int S) {
  MetaLayout L(T, S);
  SegArgs sg;
  sg.seg_starts = reinterpret_cast<const int32_t*>(meta + L.off_slot);
  sg.seg_adapter = nullptr;
  sg.n_seg = S + 1;
  return sg;
}
}  // namespace

cudaError_t launch_shrink_segment_tc(lora_dtype dt, const ShrinkArgs& a, const SegArgs& s,
                                     cudaStream_t st) {
  return shrink_tc_any(dt, a, s, st, nullptr, 0);
}

cudaError_t launch_expand_segment_tc(lora_dtype dt, const ExpandArgs& a, const SegArgs& s,
                                     cudaStream_t st) {
  return expand_tc_any(dt, a, s, st, nullptr, 0);
}

cudaError_t launch_shrink_grouped_tc(lora_dtype dt, const ShrinkArgs& a, cudaStream_t st) {
  MetaLayout L(a.T, a.S);
  return shrink_tc_any(dt, a, grouped_segments(a.meta, a.T, a.S), st,
                       reinterpret_cast<const int32_t*>(a.meta + L.off_perm), a.S);
}

cudaError_t launch_expand_grouped_tc(lora_dtype dt, const ExpandArgs& a, cudaStream_t st) {
  MetaLayout L(a.T, a.S);
  return expand_tc_any(dt, a, grouped_segments(a.meta, a.T, a.S), st,
                       reinterpret_cast<const int32_t*>(a.meta + L.off_perm), a.S);
}

}  // namespace lora
