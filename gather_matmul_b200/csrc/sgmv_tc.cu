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

// warps 0-3: loads (one per SM sub-partition, so small gathers issue four-wide),
// then the epilogue on TMEM lane quadrant = warp; warp 4: MMA issue.
constexpr int kShrThreads = 160;

template <typename E, int R>
__global__ void __launch_bounds__(kShrThreads, 2)
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
      for (int e = tid; e < valid * R; e += kShrThreads) bufs[(size_t)token(m0 + e / R) * R + e % R] = 0.f;
    return;
  }

  const int nkb_all = (P.D + kBK - 1) / kBK;
  const int kb0 = kr * nkb_all / KS, kb1 = (kr + 1) * nkb_all / KS;
  const int nkb = kb1 - kb0;                  // >= 1 (the host keeps KS <= nkb_all)

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 4);           // one arrival per load warp
      ptx::mbar_init(&empty[s], 1);          // tcgen05.commit
    }
    ptx::mbar_init(accbar, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&P.tmX);
    ptx::prefetch_tensormap(&P.tmA[slice]);
  }
  if (warp == 4) {
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
  if (warp < 4) {
    // load warps: the adapter tile and the x tile (one 2-D tile, or up to 32
    // four-row gathers, gather g issued by warp g % 4, lane g / 4)
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      if (i >= kStages) ok &= ptx::mbar_wait(&empty[s], ph ^ 1);   // MMAs of i - kStages done
      char* st = smem + (size_t)s * L::kStageBytes;
      const int kx = (kb0 + i) * kBK;
      const int mine = perm ? max((ngroups - warp + 3) / 4, 0) : 0;
      if (lane == 0) {
        uint32_t bytes = (uint32_t)(mine * 512);
        if (warp == 0) bytes += (uint32_t)L::kABytes + (perm ? 0u : (uint32_t)L::kXBytes);
        ptx::mbar_arrive_expect_tx(&full[s], bytes);
        if (warp == 0) {
          ptx::tma_load_2d(st + L::kXBytes, &P.tmA[slice], kx, adapter * R, &full[s]);
          if (!perm) ptx::tma_load_2d(st, &P.tmX, kx, m0, &full[s]);
        }
      }
      __syncwarp();
      const int g = warp + 4 * lane;
      if (perm && g < ngroups) {
        int rr[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int p = m0 + 4 * g + j;
          rr[j] = perm[p < m0 + valid ? p : m0];
        }
        ptx::tma_gather4(st + g * 4 * 128, &P.tmX, kx, rr[0], rr[1], rr[2], rr[3], &full[s]);
      }
    }
  } else if (lane == 0) {
    // MMA issuer (warp 4)
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

  // accumulator row m = 32 * warp + lane (warps 0-3), r fp32 columns
  const bool has_row = warp < 4;
  const int m = warp * 32 + lane;
  float v[R];
  if (has_row) {
#pragma unroll
    for (int c = 0; c < R / 16; ++c) {
      uint32_t r[16];
      ptx::tc_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c * 16, r);
      ptx::tc_wait_ld();
#pragma unroll
      for (int u = 0; u < 16; ++u) v[c * 16 + u] = __uint_as_float(r[u]);
    }
  }
  if (KS == 1) {
    if (has_row && m < valid) {
      float4* row = reinterpret_cast<float4*>(bufs + (size_t)token(m0 + m) * R);
#pragma unroll
      for (int q = 0; q < R / 4; ++q) row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  } else {
    // Split-K sum.  Row m belongs to rank m / rows; every rank pushes its
    // partial row into slot [kr] of the owner's receive area (the owner's
    // drained stage memory), then each owner adds its KS slots in rank order.
    const int rows = kTM / KS;
    cluster.barrier_arrive();                 // this CTA's MMAs and stages are done...
    cluster.barrier_wait();                   // ...and so are every peer's
    float* recv = reinterpret_cast<float*>(smem);
    if (has_row) {
      float* dst = cluster.map_shared_rank(recv, m / rows) + (size_t)(kr * rows + m % rows) * L::kPitch;
#pragma unroll
      for (int q = 0; q < R / 4; ++q)
        reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
    cluster.sync();                           // every partial has arrived
    for (int e = tid; e < rows * R; e += kShrThreads) {
      const int lm = e / R, j = e % R;
      float sum = 0.f;
      for (int q = 0; q < KS; ++q) sum += recv[(size_t)(q * rows + lm) * L::kPitch + j];
      const int mm = kr * rows + lm;
      if (mm < valid) bufs[(size_t)token(m0 + mm) * R + j] = sum;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 4) ptx::tmem_dealloc(tmem, kTmemCols);
  if (!ok && tid == 0) atomicAdd(P.bad_meta, 1);
}

struct ExpandTCParams {
  CUtensorMap tmB[LORA_MAX_SLICES];      // B_i as [S*D_out_i rows, r cols], box {r, 128}
  CUtensorMap tmY;                       // y as [T rows, ldy cols], box {64, 128}, 128B swizzle
  CUtensorMap tmYg;                      // y, box {64, 1}: 4-row gathers
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
  int NJ, n_chunks;                      // each CTA walks NJ consecutive 128-column tiles
  float scale;
  int* bad_index;
  int* bad_meta;
};

template <int R>
struct ExpandSmem {
  static constexpr int kYS = 3;                           // {B tile, y tile} ring stages
  static constexpr int kRowBytes = R * 2;                 // = swizzle width of the operands
  static constexpr int kBBytes = kNT * kRowBytes;
  static constexpr int kHBytes = kTM * kRowBytes;
  static constexpr int kYHalf = kTM * 128;                // 64 columns x 128 rows, 128B swizzle
  static constexpr int kYBytes = 2 * kYHalf;
  static constexpr size_t kOffB = 0;
  static constexpr size_t kOffHi = kOffB + (size_t)kYS * kBBytes;
  static constexpr size_t kOffLo = kOffHi + kHBytes;
  static constexpr size_t kOffY = kOffLo + kHBytes;
  static constexpr size_t kOffBar = kOffY + (size_t)kYS * kYBytes;
  static constexpr size_t kTotal = kOffBar + 8 * (2 * kYS + 5) + 64 + 1024;
};

// warps 0-3: epilogue (TMEM lane quadrant = warp), warps 4-7: loads (one per
// SM sub-partition, so small copies issue four-wide), warp 8: MMA issue.
constexpr int kExpThreads = 288;

template <typename E, int R>
__global__ void __launch_bounds__(kExpThreads, 1)
sgmv_expand_tc_kernel(const __grid_constant__ ExpandTCParams P) {
  using L = ExpandSmem<R>;
  constexpr int kYS = L::kYS;
  constexpr bool kBF = std::is_same<E, __nv_bfloat16>::value;
  constexpr uint32_t kIdesc = ptx::umma_idesc_f16(kBF, kTM, kNT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.y;
  const int Dout = P.D_out[slice];
  const int ntiles = (Dout + kNT - 1) / kNT;
  const int chunk = blockIdx.x % P.n_chunks;
  const int j0 = chunk * P.NJ, j1 = min(ntiles, j0 + P.NJ);
  if (j0 >= j1) return;
  const int nj = j1 - j0;

  extern __shared__ char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  char* sB = smem + L::kOffB;
  char* sHi = smem + L::kOffHi;
  char* sLo = smem + L::kOffLo;
  char* sY = smem + L::kOffY;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* empty = full + kYS;
  uint64_t* accfull = empty + kYS;       // [2]
  uint64_t* accempty = accfull + 2;      // [2]
  uint64_t* hilo = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(hilo + 1);
  int* sinfo = reinterpret_cast<int*>(tmem_slot + 4);

  if (blockIdx.x == 0 && slice == 0 && !P.implicit_slots)
    validate_segments(P.seg_starts, P.seg_adapter, P.n_seg, P.T, P.S, P.bad_index, P.bad_meta);
  const bool meta_ok = !P.implicit_slots || grouped_meta_ok(P.bad_index, P.T, P.S);
  if (warp == 0) {
    TileInfo ti;
    const bool found = meta_ok && find_tile(blockIdx.x / P.n_chunks, P.seg_starts, P.seg_adapter,
                                            P.n_seg, P.T, ti, P.implicit_slots);
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
  const int64_t ycol0 = P.y_col_off[slice];
  E* ycol = static_cast<E*>(P.y) + ycol0;
  // whole 128-row tile of consecutive tokens: y moves as 2-D TMA tiles
  const bool tiled = P.perm == nullptr && valid == kTM;

  if (tid == 0) {
    for (int s = 0; s < kYS; ++s) {
      ptx::mbar_init(&full[s], 4);       // one arrival per load warp
      ptx::mbar_init(&empty[s], 4);      // one arrival per epilogue warp
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&accfull[a], 1);
      ptx::mbar_init(&accempty[a], 4);
    }
    ptx::mbar_init(hilo, 4);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&P.tmB[slice]);
    ptx::prefetch_tensormap(tiled ? &P.tmY : &P.tmYg);
  }
  if (warp == 8) {
    ptx::tmem_alloc(tmem_slot, 2 * kNT);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp >= 4 && warp < 8) {
    // ---- loads: B tile and y tile of n-tile j into stage j % kYS
    const int pw = warp - 4;
    const int ngroups = (valid + 3) / 4;
    for (int j = 0; j < nj; ++j) {
      const int s = j % kYS;
      if (j >= kYS) ok &= ptx::mbar_wait(&empty[s], ((j / kYS) - 1) & 1);
      const int n0 = (j0 + j) * kNT;
      char* ys = sY + (size_t)s * L::kYBytes;
      // ops of this n-tile: 2 y halves x ngroups 4-row gathers, dealt out over
      // the four load warps (op o -> warp o % 4, lane o / 4)
      int my_ops = 0;
      if (!tiled)
        for (int o = pw; o < 2 * ngroups; o += 4) ++my_ops;
      const uint32_t bytes = (uint32_t)(my_ops * 512) +
                             (pw == 0 ? (uint32_t)L::kBBytes + (tiled ? (uint32_t)L::kYBytes : 0u) : 0u);
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(&full[s], bytes);
        if (pw == 0) {
          ptx::tma_load_2d(sB + (size_t)s * L::kBBytes, &P.tmB[slice], 0, adapter * Dout + n0,
                           &full[s]);
          if (tiled) {
            ptx::tma_load_2d(ys, &P.tmY, (int)(ycol0 + n0), m0, &full[s]);
            ptx::tma_load_2d(ys + L::kYHalf, &P.tmY, (int)(ycol0 + n0 + 64), m0, &full[s]);
          }
        }
      }
      __syncwarp();
      if (!tiled) {
        for (int o = pw + 4 * lane; o < 2 * ngroups; o += 128) {
          const int g = o >> 1, h = o & 1;
          int rr[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int mm = 4 * g + q < valid ? 4 * g + q : 0;
            rr[q] = P.perm ? P.perm[m0 + mm] : m0 + mm;
          }
          ptx::tma_gather4(ys + h * L::kYHalf + g * 512, &P.tmYg, (int)(ycol0 + n0 + 64 * h),
                           rr[0], rr[1], rr[2], rr[3], &full[s]);
        }
      }
    }
  } else if (warp == 8) {
    // ---- MMA issue: acc[j & 1] = hi . B^T + lo . B^T
    if (lane == 0) {
      ok &= ptx::mbar_wait(hilo, 0);
      const uint32_t hb = ptx::smem_u32(sHi), lb = ptx::smem_u32(sLo);
      for (int j = 0; j < nj; ++j) {
        const int s = j % kYS, a = j & 1;
        ok &= ptx::mbar_wait(&full[s], (j / kYS) & 1);
        if (j >= 2) ok &= ptx::mbar_wait(&accempty[a], ((j / 2) - 1) & 1);
        ptx::tc_fence_after();
        const uint32_t bb = ptx::smem_u32(sB + (size_t)s * L::kBBytes);
        const uint32_t acc = tmem + a * kNT;
#pragma unroll
        for (int ks = 0; ks < R / 16; ++ks)
          ptx::tc_mma_f16(acc, ptx::umma_desc_kmajor(hb + ks * 32, L::kRowBytes),
                          ptx::umma_desc_kmajor(bb + ks * 32, L::kRowBytes), kIdesc,
                          ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < R / 16; ++ks)
          ptx::tc_mma_f16(acc, ptx::umma_desc_kmajor(lb + ks * 32, L::kRowBytes),
                          ptx::umma_desc_kmajor(bb + ks * 32, L::kRowBytes), kIdesc, 1u);
        ptx::tc_commit(&accfull[a]);
      }
    }
  } else {
    // ---- epilogue warps 0-3: row m = TMEM lane 32 * warp + lane
    const int m = warp * 32 + lane;
    const int tok = m < valid ? (P.perm ? P.perm[m0 + m] : m0 + m) : 0;
    // row m's intermediate -> hi / lo operand rows (swizzled K-major), after an
    // exact power-of-two rescale 2^(7-e), e the exponent of max |buf| of the row
    float inv = 1.f;
    {
      const float4* brow = reinterpret_cast<const float4*>(
          P.buf + (size_t)slice * P.buf_slice_stride + (size_t)tok * R);
      float mx = 0.f;
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
      for (int c = 0; c < R / 8; ++c) {
        float4 f0 = make_float4(0.f, 0.f, 0.f, 0.f), f1 = f0;
        if (m < valid) {
          f0 = brow[2 * c];
          f1 = brow[2 * c + 1];
        }
        const float x8[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
        uint16_t hi[8], lo[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float xv = x8[u] * sc;
          hi[u] = Elem<E>::from_f32(xv);
          lo[u] = Elem<E>::from_f32(xv - Elem<E>::to_f32(hi[u]));
        }
        const int off = m * L::kRowBytes + swz<L::kRowBytes>(m, c) * 16;
        *reinterpret_cast<uint4*>(sHi + off) = *reinterpret_cast<const uint4*>(hi);
        *reinterpret_cast<uint4*>(sLo + off) = *reinterpret_cast<const uint4*>(lo);
      }
    }
    ptx::fence_proxy_async_smem();       // generic writes -> tensor-core operand reads
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(hilo);

    for (int j = 0; j < nj; ++j) {
      const int s = j % kYS, a = j & 1;
      const int n0 = (j0 + j) * kNT, nn = min(kNT, Dout - n0);
      ok &= ptx::mbar_wait(&accfull[a], (j / 2) & 1);
      ok &= ptx::mbar_wait(&full[s], (j / kYS) & 1);
      ptx::tc_fence_after();
      char* ys = sY + (size_t)s * L::kYBytes;
      // y tile layout: two 64-column halves, 128-byte rows, 16-byte chunk q of
      // a row at position q ^ (row & 7)
      for (int c = 0; c < kNT / 16; ++c) {
        uint32_t r[16];
        ptx::tc_ld16(tmem + a * kNT + ((uint32_t)(warp * 32) << 16) + c * 16, r);
        ptx::tc_wait_ld();
        if (m < valid) {
          char* hbase = ys + (c >> 2) * L::kYHalf + m * 128;
          uint4* p0 = reinterpret_cast<uint4*>(hbase + ((((2 * c) & 7)) ^ (m & 7)) * 16);
          uint4* p1 = reinterpret_cast<uint4*>(hbase + ((((2 * c + 1) & 7)) ^ (m & 7)) * 16);
          uint4 w[2] = {*p0, *p1};
          uint16_t* h = reinterpret_cast<uint16_t*>(w);
#pragma unroll
          for (int u = 0; u < 16; ++u)
            h[u] = Elem<E>::from_f32(
                fmaf(P.scale, __uint_as_float(r[u]) * inv, Elem<E>::to_f32(h[u])));
          *p0 = w[0];
          *p1 = w[1];
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&accempty[a]);   // accumulator a may be overwritten
      if (tiled && nn == kNT) {
        // whole tile: two 2-D TMA stores once all four warps updated their rows
        ptx::fence_proxy_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (warp == 0) {
          if (lane == 0) {
            ptx::tma_store_2d(&P.tmY, (int)(ycol0 + n0), m0, ys);
            ptx::tma_store_2d(&P.tmY, (int)(ycol0 + n0 + 64), m0, ys + L::kYHalf);
            ptx::bulk_commit();
            ptx::bulk_wait_read_all();                  // the stage may be refilled
          }
          __syncwarp();
        }
      } else {
        // coalesced 16-byte stores of this warp's valid rows: lane -> (row pair, chunk)
        for (int i = 0; i < 16; ++i) {
          const int mr = warp * 32 + 2 * i + (lane >> 4);
          const int q = lane & 15;
          if (mr < valid && q * 8 < nn) {
            const int tk = P.perm ? P.perm[m0 + mr] : m0 + mr;
            const uint4 v = *reinterpret_cast<const uint4*>(
                ys + (q >> 3) * L::kYHalf + mr * 128 + (((q & 7) ^ (mr & 7)) * 16));
            *reinterpret_cast<uint4*>(ycol + (size_t)tk * P.ldy + n0 + q * 8) = v;
          }
        }
        ptx::fence_proxy_async_smem();   // generic accesses before the next async refill
        __syncwarp();
      }
      if (lane == 0) ptx::mbar_arrive(&empty[s]);
    }
    if (warp == 0 && lane == 0) ptx::bulk_wait_all();
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 8) ptx::tmem_dealloc(tmem, 2 * kNT);
  if (!ok && lane == 0) atomicAdd(P.bad_meta, 1);
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
  cfg.blockDim = dim3(kShrThreads, 1, 1);
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
  {
    cudaError_t e = encode_tmap_2d(&P.tmY, dt, a.y, (uint64_t)a.ldy, (uint64_t)a.T,
                                   (uint64_t)a.ldy * 2, 64, kTM, 128);
    if (e == cudaSuccess)
      e = encode_tmap_2d(&P.tmYg, dt, a.y, (uint64_t)a.ldy, (uint64_t)a.T, (uint64_t)a.ldy * 2,
                         64, 1, 128);
    if (e != cudaSuccess) return e;
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
  // n-tiles per CTA: about three waves of one CTA per SM over all the work
  const long units = (long)max_tiles * max_nt * a.n_slices;
  int NJ = (int)((units + 3 * 148 - 1) / (3 * 148));
  NJ = NJ < 1 ? 1 : (NJ > max_nt ? max_nt : NJ);
  P.NJ = NJ;
  P.n_chunks = (max_nt + NJ - 1) / NJ;
  auto kern = sgmv_expand_tc_kernel<E, R>;
  const size_t smem = ExpandSmem<R>::kTotal;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(max_tiles * P.n_chunks, a.n_slices, 1), kExpThreads, smem, st>>>(P);
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
