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
//   (up to 16) covers the K range of one tile when tiles are too few to fill
//   the GPU.  A 4-6 stage pipeline of 64-wide K blocks: four load warps (one
//   per SM sub-partition) bring the adapter tile (r x 64) and the x tile
//   (128 x 64, 128-byte swizzle) by TMA, as one 2-D box for consecutive rows
//   or as 4-row gathers (tile::gather4) through the grouping permutation; one
//   thread issues tcgen05.mma (kind::f16, fp32 accumulator in tensor memory)
//   and tcgen05.commit frees the stage.  The accumulator is read back with
//   tcgen05.ld; split-K partials are pushed to the owning rank through
//   distributed shared memory and summed in rank order (no atomics).
// Expand  Y[rows][cols] += scale * buf[rows][:] . B[a][cols]^T   M = 128, N = 128, K = r
//   Persistent, one CTA per SM over a byte-weighted static schedule of
//   (slice, tile, 128-column) pairs (see the expand section below).  The fp32
//   intermediate enters the tensor core as hi + lo of the input type after an
//   exact power-of-two rescale per row (about 16 bits for bf16, 22 for fp16),
//   two MMAs per K step into one fp32 accumulator; a tile of at most 48 rows
//   swaps the operands.  y tiles move by 2-D TMA (consecutive rows) or 4-row
//   gathers; the epilogue adds scale * acc with one round-to-nearest-even.
//   Rows past the segment and rows without an adapter are never written.
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
constexpr int kNT = 128;          // expand output columns per CTA (MMA N)

struct TileInfo {
  int seg, m0, valid, adapter;
};

// Tile `tile` of the segment list, segments clamped into [0, T] so that no
// access can leave the buffers even for malformed lists (those are counted
// separately).  Warp-cooperative; every lane returns the same answer.
__device__ bool find_tile(int tile, const int32_t* __restrict__ ss,
                          const int32_t* __restrict__ sa, int n_seg, int T, TileInfo& ti,
                          int implicit_slots, int trows = kTM) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int s0 = 0; s0 < n_seg; s0 += 32) {
    const int s = s0 + lane;
    int a = 0, b = 0;
    if (s < n_seg) {
      a = min(max(ss[s], 0), T);
      b = max(a, min(max(ss[s + 1], 0), T));
    }
    const int nt = (b - a + trows - 1) / trows;
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
      ti.m0 = sa_l + (tile - base - excl) * trows;
      ti.valid = min(trows, sb_l - ti.m0);
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
  CUtensorMap tmA8[LORA_MAX_SLICES];     // the same, box {64, 8}: a smaller slot rank, 8 rows a copy
  const int32_t* seg_starts;
  const int32_t* seg_adapter;
  int n_seg;
  float* buf;
  const int32_t* perm;                   // row p of a tile is token perm[p]; null = identity
  const int32_t* idx;                    // per-token indices checked against the grouping
  int implicit_slots;                    // > 0: segment g is slot g (per-token grouping)
  int T, D, S, n_slices, KS;
  int trows;                             // rows per tile (<= kTM, the MMA's M)
  int* bad_index;
  int* bad_meta;
  const char* meta;                      // workspace: per-slot ranks
};

// stages of 16 KB x + r x 128 B adapter: 108 / 100 / 96 KB for r = 16 / 32 / 64,
// so that two CTAs fit per SM at every rank.  (Measured: giving a tile of few
// rows more or larger stages lets those CTAs take bandwidth from the CTAs of
// full tiles, which end the kernel, and made the large mixed batch slower.)
template <int R>
constexpr int stages_for() { return R == 16 ? 6 : (R == 32 ? 5 : 4); }

template <int R>
struct ShrinkSmem {
  static constexpr int kXBytes = kTM * 128;
  static constexpr int kABytes = R * 128;
  static constexpr int kStageBytes = kXBytes + kABytes;   // multiple of 1024
  static constexpr int kPitch = R + 4;                     // floats, partial-sum rows
  static constexpr int kStages = stages_for<R>();
  static constexpr size_t kBar = (size_t)kStageBytes * kStages;
  static constexpr size_t kTok = kBar + 8 * (2 * kStages + 1) + 64;   // int [kTM]
  static constexpr size_t kTotal = kTok + 4 * kTM + 1024;
};

static_assert(2 * (ShrinkSmem<16>::kTotal + 1024) <= 228 * 1024 &&
                  2 * (ShrinkSmem<32>::kTotal + 1024) <= 228 * 1024 &&
                  2 * (ShrinkSmem<64>::kTotal + 1024) <= 228 * 1024,
              "two shrink CTAs per SM");

// warps 0-3: loads (one per SM sub-partition, so small gathers issue four-wide),
// then the epilogue on TMEM lane quadrant = warp; warp 4: MMA issue.
constexpr int kShrThreads = 160;
// Rows per shrink tile: 96 for a per-token grouping over 64 or more slots,
// else 128 (the MMA's M either way; a 96-row tile leaves a quarter of the
// accumulator unused).  Over many slots a few popular slots' full tiles are
// the kernel's long poles; cutting them at 96 rows shortens them while the
// grid still fits one wave: large mixed batch 34.8 us against 39.2 (88 rows:
// the same, 80 or 64: 50 us, as the extra tiles no longer fit one wave).
// Batches over few slots keep 128 (96 adds empty CTAs: decode +0.3 us).
constexpr int kShrManySlots = 64, kShrRowsManySlots = 96;

template <typename E, int R>
__global__ void __launch_bounds__(kShrThreads, 2)
sgmv_shrink_tc_kernel(const __grid_constant__ ShrinkTCParams P) {
  using L = ShrinkSmem<R>;
  constexpr int kStages = L::kStages;
  constexpr bool kBF = std::is_same<E, __nv_bfloat16>::value;
  constexpr uint32_t kTmemCols = R < 32 ? 32 : R;
  ptx::grid_dep_wait();               // grouping, x and buf producers have finished
  ptx::grid_dep_launch_dependents();
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
  int* stok = reinterpret_cast<int*>(smem + L::kTok);

  if (blockIdx.x == 0 && slice == 0 && !P.implicit_slots)
    validate_segments(P.seg_starts, P.seg_adapter, P.n_seg, P.T, P.S, P.bad_index, P.bad_meta);
  if (warp == 0) {
    // the tile is looked up while the header is read (the lookup stays inside
    // the workspace whatever sizes it was built for); the grouping metadata
    // must have been built for this call's sizes
    const MetaHeader* hdr = reinterpret_cast<const MetaHeader*>(P.meta);
    const int hT = P.implicit_slots ? hdr->T : P.T, hS = P.implicit_slots ? hdr->S : P.S;
    const int has_ranks = hdr->has_ranks;
    TileInfo ti;
    const bool found = find_tile(blockIdx.x / KS, P.seg_starts, P.seg_adapter, P.n_seg, P.T, ti,
                                 P.implicit_slots, P.trows);
    const bool meta_ok = hT == P.T && hS == P.S;
    if (!meta_ok && lane == 0 && blockIdx.x == 0 && slice == 0) atomicAdd(P.bad_meta, 1);
    if (lane == 0) {
      sinfo[0] = found && meta_ok ? 1 : 0;
      sinfo[1] = ti.m0;
      sinfo[2] = ti.valid;
      sinfo[3] = ti.adapter;
      // the slot's own rank (a multiple of 8, or R)
      sinfo[4] = has_ranks && found && meta_ok ? slot_rank(P.meta, P.S, ti.adapter, R) : R;
    }
  }
  __syncthreads();
  if (!sinfo[0]) return;                      // same for the whole cluster
  const int m0 = sinfo[1], valid = sinfo[2], adapter = sinfo[3];
  float* bufs = P.buf + (size_t)slice * P.T * R;
  const int32_t* perm = P.perm;
  // token of tile row p, or -1 when a per-token grouping placed a token whose
  // index disagrees with the group (stale workspace): that row is not written,
  // and the writer of the row counts it
  auto token = [&](int p, bool count) {
    if (!perm) return p;
    const int t = perm[p];
    if (grouped_row_ok(P.idx, t, adapter, P.S)) return t;
    if (count && slice == 0) atomicAdd(P.bad_meta, 1);
    return -1;
  };
  if (adapter < 0 || adapter >= P.S) {        // no adapter: zero rows (rank 0 writes them)
    if (kr == 0)
      for (int m = tid; m < valid; m += kShrThreads) {
        const int t = token(m0 + m, true);
        if (t >= 0) {
          float4* row = reinterpret_cast<float4*>(bufs + (size_t)t * R);
#pragma unroll
          for (int q = 0; q < R / 4; ++q) row[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    return;
  }

  const int nkb_all = (P.D + kBK - 1) / kBK;
  const int kb0 = kr * nkb_all / KS, kb1 = (kr + 1) * nkb_all / KS;
  const int nkb = kb1 - kb0;                  // >= 1 (the host keeps KS <= nkb_all)
  // the slot's own rank kk (a multiple of 8): only its first kk rows of A are
  // read, and the MMA is N = kk rounded up to 16 wide
  const int kk = sinfo[4];
  const uint32_t idesc = ptx::umma_idesc_f16(kBF, kTM, kk < 16 ? 16 : (kk + 15) & ~15);
  const uint32_t a_bytes = (uint32_t)kk * 128;

  const int ngroups = (valid + 3) / 4;        // 4-row gathers per stage (row indirection)
  // load warps: gather g = warp + 4 * lane brings tile rows 4g..4g+3; their
  // tokens are the same at every K step, so they are read once, here, while
  // the barriers and tensor memory are set up
  const int g = warp + 4 * lane;
  int rr[4] = {0, 0, 0, 0};
  if (warp < 4 && perm && g < ngroups) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = m0 + 4 * g + j;
      rr[j] = perm[p < m0 + valid ? p : m0];
    }
  }
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
        if (warp == 0) bytes += a_bytes + (perm ? 0u : (uint32_t)L::kXBytes);
        ptx::mbar_arrive_expect_tx(&full[s], bytes);
        if (warp == 0) {
          if (kk == R) {
            ptx::tma_load_2d(st + L::kXBytes, &P.tmA[slice], kx, adapter * R, &full[s]);
          } else {
            for (int b = 0; b < kk / 8; ++b)       // same layout as one kk-row box
              ptx::tma_load_2d(st + L::kXBytes + b * 1024, &P.tmA8[slice], kx,
                               adapter * R + 8 * b, &full[s]);
          }
          if (!perm) ptx::tma_load_2d(st, &P.tmX, kx, m0, &full[s]);
        }
      }
      __syncwarp();
      if (perm && g < ngroups)
        ptx::tma_gather4(st + g * 4 * 128, &P.tmX, kx, rr[0], rr[1], rr[2], rr[3], &full[s]);
    }
    // while the MMAs run: the token of each tile row, checked against the
    // batch's indices, for the epilogue; a stale row is counted by the rank
    // that writes it
    const int m = warp * 32 + lane;
    stok[m] = m < valid ? token(m0 + m, KS == 1 || m / ((valid + KS - 1) / KS) == kr) : -1;
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
                        ptx::umma_desc_kmajor(aa + k * 32, 128), idesc, (i > 0 || k > 0) ? 1u : 0u);
      ptx::tc_commit(&empty[s]);              // stage s is free once these MMAs finish
    }
    ptx::tc_commit(accbar);
  }
  ok &= ptx::mbar_wait(accbar, 0);
  ptx::tc_fence_after();
  // split K: this CTA's MMAs are done, so its stages are drained and may take
  // the peers' partials; the barrier's latency overlaps the accumulator read
  if (KS > 1) cluster.barrier_arrive();

  // accumulator row m = 32 * warp + lane (warps 0-3), r fp32 columns
  const bool has_row = warp < 4;
  const int m = warp * 32 + lane;
  float v[R];
  if (has_row) {
    uint32_t r[R];
#pragma unroll
    for (int c = 0; c < R / 16; ++c) ptx::tc_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c * 16, r + c * 16);
    ptx::tc_wait_ld();
    // columns past the slot's rank: zero (the accumulator holds nothing there)
#pragma unroll
    for (int u = 0; u < R; ++u) v[u] = u < kk ? __uint_as_float(r[u]) : 0.f;
  }
  if (KS == 1) {
    const int t = has_row ? stok[m] : -1;
    if (t >= 0) {
      float4* row = reinterpret_cast<float4*>(bufs + (size_t)t * R);
#pragma unroll
      for (int q = 0; q < R / 4; ++q) row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  } else {
    // Split-K sum over the tile's valid rows: row m belongs to rank m / rpr;
    // every rank pushes its partial of the row into slot [kr] of the owner's
    // receive area (the owner's drained stage memory), then each owner adds
    // its KS slots in rank order.
    const int rpr = (valid + KS - 1) / KS;
    cluster.barrier_wait();                   // every peer's MMAs and stages are done
    float* recv = reinterpret_cast<float*>(smem);
    if (has_row && m < valid) {
      float* dst = cluster.map_shared_rank(recv, m / rpr) + (size_t)(kr * rpr + m % rpr) * L::kPitch;
#pragma unroll
      for (int q = 0; q < R / 4; ++q)
        reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
    cluster.sync();                           // every partial has arrived
    // four columns of an owned row per step, every partial loaded first
    const int own0 = kr * rpr, nown = max(0, min(rpr, valid - own0));
    const float4* rv = reinterpret_cast<const float4*>(recv);
    for (int e = tid; e < nown * (R / 4); e += kShrThreads) {
      const int lm = e / (R / 4), c = e % (R / 4);
      float4 part[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q < KS) part[q] = rv[(size_t)(q * rpr + lm) * (L::kPitch / 4) + c];
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q < KS) {
          sum.x += part[q].x;
          sum.y += part[q].y;
          sum.z += part[q].z;
          sum.w += part[q].w;
        }
      const int t = stok[own0 + lm];
      if (t >= 0) reinterpret_cast<float4*>(bufs + (size_t)t * R)[c] = sum;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 4) ptx::tmem_dealloc(tmem, kTmemCols);
  if (!ok && tid == 0) atomicAdd(P.bad_meta, 1);
}

constexpr int kMaxSegTC = 2048;          // longer segment lists use the item kernels
constexpr int kMaxSegChunks = kMaxSegTC / 32 + 1;
constexpr int kSegCache = 256;           // segment lists up to this long are read once

struct SegView {
  const int32_t* ss;
  const int32_t* sa;
  int n_seg, T, S, implicit_slots;
  int4* cache;                           // shared-memory copy of the first kSegCache segments
  // the same, from the copy when the whole list is in it; kc = the adapter's
  // rank class from the copy, or -1 when it is not cached
  __device__ __forceinline__ void get_cached(int s, int& a, int& b, int& ad, int& kc) const {
    if (n_seg <= kSegCache) {
      const int4 c = s < n_seg ? cache[s] : make_int4(0, 0, -1, 0);
      a = c.x; b = c.y; ad = c.z; kc = c.w;
    } else {
      get(s, a, b, ad);
      kc = -1;
    }
  }
  // segment s clamped into [0, T]; adapter -1 when it has none or is out of range
  __device__ __forceinline__ void get(int s, int& a, int& b, int& ad) const {
    a = 0; b = 0; ad = -1;
    if (s < n_seg) {
      a = min(max(ss[s], 0), T);
      b = max(a, min(max(ss[s + 1], 0), T));
      ad = implicit_slots ? (s < implicit_slots ? s : -1) : sa[s];
      if (ad < 0 || ad >= S) ad = -1;
    }
  }
};

// min(ceil(num / w), nt) for a pair weight w: 32-bit arithmetic once the
// quotient is known to be below nt (nt * w stays far below 2^32), instead of
// a 64-bit division
__device__ __forceinline__ int ceil_pos_nt(int64_t num, int w, int nt) {
  if (num <= 0) return 0;
  if (num >= (int64_t)nt * w) return nt;
  return (int)(((uint32_t)num + (uint32_t)w - 1u) / (uint32_t)w);
}

// ---------------------------------------------------------------- expand
// Persistent: one CTA per SM walks a contiguous range of (slice, tile, n-tile)
// pairs.  The pairs are ordered slice-major, then by tile, then by 128-column
// output tile, and weighted by the bytes they move (B tile + y rows read and
// written + a fixed cost), so every CTA gets the same share of the traffic
// whatever the mix of full and nearly empty tiles.  A CTA lists its tile runs
// (a tile and the n-tiles of it that fall in its range) once, then runs one
// continuous pipeline over them:
//   load warps   B tile + y tile of each pair into a ring of stages; the
//                hi / lo operand of each run (double-buffered)
//   MMA warp     acc = hi . B^T + lo . B^T into one of two TMEM accumulators;
//                a tile of <= swap_max<R>() rows swaps the operands (M = 128 output
//                columns, N = its rows rounded to 16) so the epilogue only
//                touches the rows that exist
//   epilogue     y += scale * acc, one rounding; two warps per TMEM lane
//                quadrant split the columns (or the token chunks)
struct ExpRun {
  int m0, valid, adapter, slice, j0, j1;
  int kc;        // the adapter's rank rounded up to 16 << kc (per-slot ranks)
};
constexpr int kMaxRuns = 64;
// Tiles of at most swap_max<R>() rows swap operands.  Measured on B200 (one
// lora_bgmv step): at rank 32, 48 rows (large mixed 97.2 us against 97.5 with
// 56 and 97.6 with 64); at rank 64, 64 rows (decode qkv / gate_up / down
// 25.8 / 37.6 / 25.1 us against 26.7 / 39.6 / 26.3 with 48; 56 the same).
template <int R>
constexpr int swap_max() { return R >= 64 ? 64 : 48; }

struct ExpandTCParams {
  // B_i as [S*D_out_i rows, r cols], box {16 << c, 128} with a (32 << c)-byte
  // swizzle: class c = 0, 1, 2 reads the first 16 / 32 / 64 columns of each
  // row (a slot's own rank rounded up to 16; c <= log2(r / 16))
  CUtensorMap tmB[3][LORA_MAX_SLICES];
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
  const int32_t* idx;                    // per-token indices checked against the grouping
  int implicit_slots;                    // > 0: segment g is slot g (per-token grouping)
  int T, S, n_slices;
  float scale;
  int* bad_index;
  int* bad_meta;
  const char* meta;                      // workspace: per-slot ranks
  int early;                             // wait for the previous kernel only before reading buf
};

template <int R>
struct ExpandSmem {
  static constexpr int kRowBytes = R * 2;                 // = swizzle width of the operands
  static constexpr int kBBytes = kNT * kRowBytes;
  static constexpr int kHBytes = kTM * kRowBytes;
  static constexpr int kYHalf = kTM * 128;                // 64 columns x 128 rows, 128B swizzle
  static constexpr int kYBytes = 2 * kYHalf;
  static constexpr int kYS = R == 64 ? 3 : (R == 32 ? 4 : 5);   // {B tile, y tile} stages
  static constexpr size_t kOffY = 0;
  static constexpr size_t kOffB = kOffY + (size_t)kYS * kYBytes;
  static constexpr size_t kOffHL = kOffB + (size_t)kYS * kBBytes;     // [2] x {hi, lo}
  static constexpr size_t kOffInv = kOffHL + 4 * (size_t)kHBytes;     // float [2][128]
  static constexpr size_t kOffTok = kOffInv + 2 * kTM * 4;            // int [2][128]
  static constexpr size_t kOffRun = kOffTok + 2 * kTM * 4;            // ExpRun [kMaxRuns]
  static constexpr size_t kOffChunk = kOffRun + kMaxRuns * sizeof(ExpRun);   // int64 [chunks]
  static constexpr size_t kOffSeg = (kOffChunk + 8 * kMaxSegChunks + 15) & ~size_t(15);   // int4 [kSegCache]
  static constexpr size_t kOffBar = kOffSeg + 16 * kSegCache;
  static constexpr int kNBar = 2 * kYS + 10;
  static constexpr size_t kOffMisc = kOffBar + 8 * kNBar;             // tmem, n_runs, next
  static constexpr size_t kTotal = kOffMisc + 64 + 1024;
  static_assert(kOffB % 1024 == 0 && kOffHL % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kOffInv % 16 == 0 && kOffTok % 16 == 0 && kOffRun % 8 == 0, "alignment");
  static_assert(kOffChunk % 8 == 0 && kOffSeg % 16 == 0 && kOffBar % 8 == 0, "alignment");
};

// The time a pair takes on one SM, in quarter nanoseconds, from
// least-squares fits on B200 of each CTA's time against its pairs, their
// rows and its runs (residual 0.2-1.9 us per CTA):
//   rank 16 and 32 (a fit over Zipf, uniform, mixed-size, prefill and
//     fused-slice decode batches):
//     operand-swapped tile (<= swap_max<R>() rows): 0.47 us + 16.4 ns per valid
//     row (its epilogue is one round of the pipeline for few rows);
//     128-row layout (more rows): 1.56 us + 1.3 ns per valid row, nearly
//     flat (the whole tile passes through tensor memory and the epilogue);
//   rank 64: the weights of an earlier fit (0.58 us + 16.5 ns, 1.2 us +
//     5 ns), which a simulation of the schedule with a rank-64 fit's costs
//     found as good as any refit (the refit above made the decode gate_up
//     expand 30.1 -> 31.6 us);
//   plus about 4.5 ns per rank column of the B tile (its 256 r bytes).
// With the earlier weights at rank 32 the CTAs of partial 128-row tiles ran
// 20 % longer than the mean on the large mixed batch (62 against 52 us);
// refitted, the large mixed expand went from 66.4 to 64.1 us (a rank-32-only
// fit: 65.2 us).  Weights in bytes moved had rated a full tile at 3.3 small
// tiles and a 90-row tile far below a full one, which left CTAs of small
// groups as the long poles.
template <int R>
__device__ __forceinline__ int64_t pair_weight(int valid) {
  constexpr int kSwapMax = swap_max<R>();
  if constexpr (R >= 64)
    return valid <= kSwapMax ? 1744 + 18 * R + 66 * (int64_t)valid
                             : 4224 + 18 * R + 20 * (int64_t)valid;
  else
    return valid <= kSwapMax ? 1320 + 18 * R + 66 * (int64_t)valid
                             : 5660 + 18 * R + 5 * (int64_t)valid;
}

// Per n-tile weight of one segment: its full tiles and its partial last tile.
template <int R>
__device__ __forceinline__ int64_t seg_weight(int a, int b, int ad) {
  if (ad < 0) return 0;
  const int len = b - a;
  const int rem = len % kTM;
  return (int64_t)(len / kTM) * pair_weight<R>(kTM) + (rem ? pair_weight<R>(rem) : 0);
}

// Rank class of an adapter: its rank rounded up to 16 << kc (the call's rank
// when the workspace holds no per-slot ranks; nothing is read then).
template <int R>
__device__ __forceinline__ int rank_class(const char* meta, int S, int adapter, int has_ranks) {
  const int k = has_ranks ? slot_rank(meta, S, adapter, R) : R;
  const int k16 = max(16, (k + 15) & ~15);
  return k16 == 16 ? 0 : (k16 == 32 ? 1 : 2);
}

// Warp 0 of the CTA: per-chunk (32 segments) weights into chunkW, total
// returned in every lane; the first kSegCache segments and their adapters'
// rank classes are copied to shared memory.
template <int R>
__device__ int64_t seg_chunk_weights(const SegView& sv, int64_t* chunkW, const char* meta,
                                     int has_ranks) {
  const int lane = threadIdx.x & 31;
  const int nch = (sv.n_seg + 31) / 32;
  int64_t total = 0;
  // four chunks per round: all their segment loads first (ahead of the
  // shared-memory copies, which the compiler may not move loads across),
  // then the weights and the reductions
  constexpr int kU = 4;
  for (int c0 = 0; c0 < nch; c0 += kU) {
    int64_t w[kU];
    int a[kU], b[kU], ad[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) sv.get((c0 + u) * 32 + lane, a[u], b[u], ad[u]);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int sidx = (c0 + u) * 32 + lane;
      if (sidx < kSegCache)
        sv.cache[sidx] = make_int4(a[u], b[u], ad[u],
                                   ad[u] >= 0 ? rank_class<R>(meta, sv.S, ad[u], has_ranks) : 0);
      w[u] = seg_weight<R>(a[u], b[u], ad[u]);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      int64_t v = w[u];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && c0 + u < nch) chunkW[c0 + u] = v;
      total += c0 + u < nch ? v : 0;
    }
  }
  return total;
}


// Warp-cooperative: the tile runs whose pair start positions fall in
// [lo, hi), in schedule order, at most kMaxRuns of them.  Returns the count;
// *next is hi when the list is complete, else where the next list starts.
template <int R>
__device__ int build_runs(const SegView& sv, const int64_t* chunkW, int64_t Wt,
                          const int* ntiles, int n_slices, int64_t lo, int64_t hi,
                          ExpRun* runs, int64_t* next, const char* meta, int has_ranks) {
  const int lane = threadIdx.x & 31;
  const int nch = (sv.n_seg + 31) / 32;
  int n = 0;
  int64_t pos = 0;
  *next = hi;
  for (int i = 0; i < n_slices && pos < hi; ++i) {
    const int64_t nt = ntiles[i];
    if (pos + nt * Wt <= lo) {
      pos += nt * Wt;
      continue;
    }
    int64_t cpos = pos;
    for (int c = 0; c < nch && cpos < hi; ++c) {
      const int64_t cw = nt * chunkW[c];
      if (cpos + cw <= lo || cw == 0) {
        cpos += cw;
        continue;
      }
      int a, b, ad, kc;
      sv.get_cached(c * 32 + lane, a, b, ad, kc);
      const int64_t sw = nt * seg_weight<R>(a, b, ad);
      int64_t incl = sw;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int64_t spos = cpos + incl - sw;
      unsigned mask = __ballot_sync(0xffffffffu, sw > 0 && spos < hi && spos + sw > lo);
      while (mask) {
        const int l = __ffs(mask) - 1;
        mask &= mask - 1;
        const int a_l = __shfl_sync(0xffffffffu, a, l);
        const int len = __shfl_sync(0xffffffffu, b, l) - a_l;
        const int ad_l = __shfl_sync(0xffffffffu, ad, l);
        const int64_t sp = __shfl_sync(0xffffffffu, spos, l);
        const int kc_c = __shfl_sync(0xffffffffu, kc, l);
        const int kc_l = kc_c >= 0 ? kc_c : rank_class<R>(meta, sv.S, ad_l, has_ranks);
        const int ntk = (len + kTM - 1) / kTM;
        for (int k0 = 0; k0 < ntk; k0 += 32) {
          const int k = k0 + lane;
          const int valid = k < ntk ? min(kTM, len - k * kTM) : 0;
          const int w = (int)pair_weight<R>(valid);
          const int64_t tpos = sp + nt * (int64_t)k * pair_weight<R>(kTM);
          const int jl = ceil_pos_nt(lo - tpos, w, (int)nt);
          const int jh = ceil_pos_nt(hi - tpos, w, (int)nt);
          const bool has = k < ntk && jl < jh;
          const unsigned hm = __ballot_sync(0xffffffffu, has);
          const int rank = __popc(hm & ((1u << lane) - 1));
          if (has && n + rank < kMaxRuns)
            runs[n + rank] = ExpRun{a_l + k * kTM, valid, ad_l, i, jl, jh, kc_l};
          const int cnt = __popc(hm);
          if (n + cnt > kMaxRuns) {
            // the first run that did not fit starts the next list
            const int64_t resume = max(lo, tpos);
            const unsigned over = __ballot_sync(0xffffffffu, has && n + rank == kMaxRuns);
            *next = __shfl_sync(0xffffffffu, resume, __ffs(over) - 1);
            return kMaxRuns;
          }
          n += cnt;
        }
      }
      cpos += cw;
    }
    pos += nt * Wt;
  }
  return n;
}

// warps 0-7: epilogue (TMEM lane quadrant = warp % 4, column half = warp / 4),
// warps 8-11: loads (one per SM sub-partition), warp 12: MMA issue, warps
// 13-: operands (each run's tokens and hi / lo rows, one run ahead): two
// warps reading two buf rows per lane at once up to rank 32; at rank 64 (a
// row fills half the registers) three warps reading one row per lane at a
// time, so the rows of a run of up to 96 tokens are read in one round.
constexpr int kExpLoad0 = 8, kExpMma = 12, kExpOpnd0 = 13;
template <int R>
constexpr int exp_opnd_warps() { return R >= 64 ? 3 : 2; }
template <int R>
constexpr int exp_threads() { return 32 * (kExpOpnd0 + exp_opnd_warps<R>()); }

template <typename E, int R>
__global__ void __launch_bounds__(exp_threads<R>(), 1)
sgmv_expand_tc_kernel(const __grid_constant__ ExpandTCParams P) {
  using L = ExpandSmem<R>;
  constexpr int kYS = L::kYS;
  constexpr int kSwapMax = swap_max<R>();
  constexpr int kOW = exp_opnd_warps<R>();             // operand warps
  constexpr int kRPL = (kTM + 32 * kOW - 1) / (32 * kOW);  // operand rows per lane
  constexpr bool kBF = std::is_same<E, __nv_bfloat16>::value;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // The previous kernel (programmatic dependent launch) is waited for here,
  // or, when it is known to be the shrink of the same batch, only by the load
  // warps before their first buf read: the run lists, the B tiles and the y
  // tiles of the first pairs are then set up while the shrink finishes.
  if (!P.early) ptx::grid_dep_wait();
  ptx::grid_dep_launch_dependents();

  extern __shared__ char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  char* sY = smem + L::kOffY;
  char* sB = smem + L::kOffB;
  char* sHL = smem + L::kOffHL;
  float* sInv = reinterpret_cast<float*>(smem + L::kOffInv);
  int* sTok = reinterpret_cast<int*>(smem + L::kOffTok);
  ExpRun* runs = reinterpret_cast<ExpRun*>(smem + L::kOffRun);
  int64_t* chunkW = reinterpret_cast<int64_t*>(smem + L::kOffChunk);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* empty = full + kYS;
  uint64_t* accfull = empty + kYS;       // [2]
  uint64_t* accempty = accfull + 2;      // [2]
  uint64_t* hlfull = accempty + 2;       // [2]
  uint64_t* hlempty = hlfull + 2;        // [2]
  uint64_t* tokfull = hlempty + 2;       // [2] tokens of operand buffer b written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  int* sNRuns = reinterpret_cast<int*>(tmem_slot + 1);
  int64_t* sRange = reinterpret_cast<int64_t*>(smem + L::kOffMisc + 8);   // lo, hi, Wt, next
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 48);

  const SegView sv{P.seg_starts, P.seg_adapter, P.n_seg, P.T, P.S, P.implicit_slots,
                   reinterpret_cast<int4*>(smem + L::kOffSeg)};
  if (blockIdx.x == 0 && !P.implicit_slots)
    validate_segments(P.seg_starts, P.seg_adapter, P.n_seg, P.T, P.S, P.bad_index, P.bad_meta);
  int ntiles[LORA_MAX_SLICES];
  int64_t sum_nt = 0;
  for (int i = 0; i < P.n_slices; ++i) {
    ntiles[i] = (P.D_out[i] + kNT - 1) / kNT;
    sum_nt += ntiles[i];
  }

  int has_ranks = 0;                     // read by the MMA warp, which builds the run lists
  if (warp == kExpMma) {
    ptx::tmem_alloc(tmem_slot, 2 * kNT);
    ptx::tmem_relinquish();
    // this CTA's share of the weighted pair sequence (the segment reads stay in
    // bounds whatever the workspace holds, so they are made while the header
    // is read)
    const MetaHeader* hdr = reinterpret_cast<const MetaHeader*>(P.meta);
    const int hT = P.implicit_slots ? hdr->T : P.T, hS = P.implicit_slots ? hdr->S : P.S;
    has_ranks = hdr->has_ranks;
    const int64_t Wt0 = seg_chunk_weights<R>(sv, chunkW, P.meta, has_ranks);
    const bool meta_ok = hT == P.T && hS == P.S;
    if (!meta_ok && lane == 0 && blockIdx.x == 0) atomicAdd(P.bad_meta, 1);
    const int64_t Wt = meta_ok ? Wt0 : 0;
    const int64_t W = Wt * sum_nt;
    if (lane == 0) {
      // CTA b takes [W F(b/G), W F((b+1)/G)).  Behind the library's own shrink
      // the CTAs start as the shrink's CTAs leave their SMs, in block order,
      // so at rank <= 32 the shares fall off linearly from 1 + 1/16 to
      // 1 - 1/16 of the mean: F(x) = x + x (1 - x) / 16 (measured on B200:
      // large mixed step 97.2 -> 96.3 us; 1/32: 96.6, 1/8: 98.3; at rank 64
      // and alone the even split is as good or better)
      const int64_t G = gridDim.x, b0 = blockIdx.x, b1 = blockIdx.x + 1;
      const bool skew = P.early && R <= 32;
      auto part = [&](int64_t b) {
        const int64_t e = W * b / G;
        return e + (skew ? e * (G - b) / G / 16 : 0);
      };
      sRange[0] = part(b0);
      sRange[1] = part(b1);
      sRange[2] = Wt;
    }
    __syncwarp();
  }
  if (tid == 0) {
    *sAbort = 0;
    for (int s = 0; s < kYS; ++s) {
      ptx::mbar_init(&full[s], 4);       // one arrival per load warp
      ptx::mbar_init(&empty[s], 8);      // one arrival per epilogue warp
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&accfull[a], 1);
      ptx::mbar_init(&accempty[a], 8);
      ptx::mbar_init(&hlfull[a], kOW);     // one arrival per operand warp
      ptx::mbar_init(&tokfull[a], kOW);
      ptx::mbar_init(&hlempty[a], 8);
    }
    ptx::fence_mbar_init();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int64_t lo = sRange[0];
  const int64_t hi = sRange[1], Wt = sRange[2];
  bool ok = true;
  // pipeline positions, continued across run lists: pair p, run u
  int p = 0, u = 0;
  // epilogue: a TMA store of half h whose stage is released once it was read
  int deferred = -1;

  while (lo < hi) {
    if (warp == kExpMma) {
      int64_t nx;
      const int n = build_runs<R>(sv, chunkW, Wt, ntiles, P.n_slices, lo, hi, runs, &nx, P.meta,
                                  has_ranks);
      if (lane == 0) {
        *sNRuns = n;
        sRange[3] = nx;
      }
    }
    __syncthreads();
    const int n_runs = *sNRuns;
    const int64_t next_lo = sRange[3];

    if (warp >= kExpLoad0 && warp < kExpMma) {
      // ---------------- loads: per pair its B tile and y rows
      const int pw = warp - kExpLoad0;
      int pl = p, ul = u;
      for (int ri = 0; ri < n_runs; ++ri, ++ul) {
        const ExpRun rn = runs[ri];
        const int hb = ul & 1;
        // the run's tokens (written by the operand warps)
        ok &= ptx::mbar_wait_ff(&tokfull[hb], (ul >> 1) & 1, sAbort);
        const int* toks = sTok + hb * kTM;
        const int Dout = P.D_out[rn.slice];
        const int64_t ycol0 = P.y_col_off[rn.slice];
        const bool tiled = P.perm == nullptr && rn.valid == kTM;
        const int ngroups = (rn.valid + 3) / 4;
        int my_ops = 0;
        if (!tiled)
          for (int o = pw; o < 2 * ngroups; o += 4) ++my_ops;
        for (int j = rn.j0; j < rn.j1; ++j, ++pl) {
          const int s = pl % kYS;
          if (pl >= kYS) ok &= ptx::mbar_wait_ff(&empty[s], ((pl / kYS) - 1) & 1, sAbort);
          const int n0 = j * kNT;
          char* ys = sY + (size_t)s * L::kYBytes;
          // the B tile holds only the first 16 << kc columns of each row
          const uint32_t bbytes = (uint32_t)(kNT * (16 << rn.kc) * 2);
          const uint32_t bytes =
              (uint32_t)(my_ops * 512) +
              (pw == 0 ? bbytes + (tiled ? (uint32_t)L::kYBytes : 0u) : 0u);
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(&full[s], bytes);
            if (pw == 0) {
              ptx::tma_load_2d(sB + (size_t)s * L::kBBytes, &P.tmB[rn.kc][rn.slice], 0,
                               rn.adapter * Dout + n0, &full[s]);
              if (tiled) {
                ptx::tma_load_2d(ys, &P.tmY, (int)(ycol0 + n0), rn.m0, &full[s]);
                ptx::tma_load_2d(ys + L::kYHalf, &P.tmY, (int)(ycol0 + n0 + 64), rn.m0, &full[s]);
              }
            }
          }
          __syncwarp();
          if (!tiled) {
            // 2 halves x ngroups 4-row gathers: op o -> warp o % 4, lane o / 4
            for (int o = pw + 4 * lane; o < 2 * ngroups; o += 128) {
              const int g = o >> 1, h = o & 1;
              int rr[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int t = toks[4 * g + q < rn.valid ? 4 * g + q : 4 * g];
                rr[q] = t >= 0 ? t : -2 - t;
              }
              ptx::tma_gather4(ys + h * L::kYHalf + g * 512, &P.tmYg, (int)(ycol0 + n0 + 64 * h),
                               rr[0], rr[1], rr[2], rr[3], &full[s]);
            }
          }
        }
      }
    } else if (warp >= kExpOpnd0) {
      // ---------------- operands: per run its tokens, then the hi / lo rows
      // of its buf rows, while the loads, MMAs and epilogue of the run before
      // are under way (double-buffered)
      const int ow = warp - kExpOpnd0;
      int ul = u;
      bool buf_ready = !P.early;
      for (int ri = 0; ri < n_runs; ++ri, ++ul) {
        const ExpRun rn = runs[ri];
        const int hb = ul & 1;
        if (ul >= 2) ok &= ptx::mbar_wait_ff(&hlempty[hb], ((ul >> 1) - 1) & 1, sAbort);
        // rows the MMA reads: all 128 in the 128-row layout, the valid rows
        // rounded up to 16 when the operands are swapped
        const int nrows = rn.valid <= kSwapMax ? (rn.valid + 15) & ~15 : kTM;
        // sTok: the row's token; -1 past the tile; -2 - token for a token whose
        // index disagrees with its group (stale workspace): still a valid row
        // address for the gathers, but never written back (counted below).
        // The gathers need only the tokens, so the index check is made after
        // they are published, together with the buf row read.
        int tk[kRPL];
#pragma unroll
        for (int i = 0; i < kRPL; ++i) {
          const int m = 32 * (ow + kOW * i) + lane;   // rows past 127 are not read
          tk[i] = m < rn.valid ? (P.perm ? P.perm[rn.m0 + m] : rn.m0 + m) : -1;
          if (m < nrows) sTok[hb * kTM + m] = tk[i];
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&tokfull[hb]);
        if (!buf_ready) {
          ptx::grid_dep_wait();                      // the shrink has written buf
          buf_ready = true;
        }
        // hi / lo after an exact power-of-two rescale 2^(7-e) (e = exponent of
        // the row's max |buf|), and the inverse scale; rows are read kB at a time
        constexpr int kB = R <= 32 ? kRPL : 1;
        char* hiP = sHL + (size_t)(2 * hb) * L::kHBytes;
        char* loP = hiP + L::kHBytes;
#pragma unroll
        for (int i0 = 0; i0 < kRPL; i0 += kB) {
          float4 f[kB][R / 4];
#pragma unroll
          for (int b = 0; b < kB; ++b) {
            const int m = 32 * (ow + kOW * (i0 + b)) + lane;
            const int tok = tk[i0 + b];
            const float4* brow = reinterpret_cast<const float4*>(
                P.buf + (size_t)rn.slice * P.buf_slice_stride + (size_t)(tok < 0 ? 0 : tok) * R);
#pragma unroll
            for (int q = 0; q < R / 4; ++q)
              f[b][q] = (m < nrows && tok >= 0 && 4 * q < (16 << rn.kc))
                            ? brow[q] : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int b = 0; b < kB; ++b) {
            const int m = 32 * (ow + kOW * (i0 + b)) + lane;
            const int tok = tk[i0 + b];
            if (m >= nrows) continue;
            const bool stale = tok >= 0 && P.perm && !grouped_row_ok(P.idx, tok, rn.adapter, P.S);
            float mx = 0.f;
#pragma unroll
            for (int q = 0; q < R / 4; ++q)
              mx = fmaxf(fmaxf(fmaxf(mx, fabsf(f[b][q].x)), fmaxf(fabsf(f[b][q].y), fabsf(f[b][q].z))),
                         fabsf(f[b][q].w));
            int e = ((__float_as_int(mx) >> 23) & 0xff) - 127;
            e = (mx > 0.f && e > -100 && e < 100) ? e : 0;
            const float sc = __int_as_float((127 - e + 7) << 23);
#pragma unroll
            for (int c = 0; c < R / 8; ++c) {
              const float x8[8] = {f[b][2 * c].x, f[b][2 * c].y, f[b][2 * c].z, f[b][2 * c].w,
                                   f[b][2 * c + 1].x, f[b][2 * c + 1].y, f[b][2 * c + 1].z,
                                   f[b][2 * c + 1].w};
              uint16_t h8[8], l8[8];
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                const float xv = x8[v] * sc;
                h8[v] = Elem<E>::from_f32(xv);
                l8[v] = Elem<E>::from_f32(xv - Elem<E>::to_f32(h8[v]));
              }
              const int off = m * L::kRowBytes + swz<L::kRowBytes>(m, c) * 16;
              *reinterpret_cast<uint4*>(hiP + off) = *reinterpret_cast<const uint4*>(h8);
              *reinterpret_cast<uint4*>(loP + off) = *reinterpret_cast<const uint4*>(l8);
            }
            sInv[hb * kTM + m] = __int_as_float((127 + e - 7) << 23);
            if (stale) {
              if (rn.j0 == 0) atomicAdd(P.bad_meta, 1);
              sTok[hb * kTM + m] = -2 - tok;   // the gathers read either form as row tok
            }
          }
        }
        ptx::fence_proxy_async_smem();   // generic writes -> tensor-core operand reads
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&hlfull[hb]);   // one arrival per operand warp
      }
    } else if (warp == kExpMma) {
      // ---------------- MMA issue
      if (lane == 0) {
        int pl = p, ul = u;
        for (int ri = 0; ri < n_runs; ++ri, ++ul) {
          const ExpRun rn = runs[ri];
          const int hb = ul & 1;
          const bool swap = rn.valid <= kSwapMax;
          const uint32_t idesc =
              ptx::umma_idesc_f16(kBF, kTM, swap ? (rn.valid + 15) / 16 * 16 : kNT);
          ok &= ptx::mbar_wait_ff(&hlfull[hb], (ul >> 1) & 1, sAbort);
          const uint32_t hiA = ptx::smem_u32(sHL + (size_t)(2 * hb) * L::kHBytes);
          const uint32_t loA = hiA + L::kHBytes;
          for (int j = rn.j0; j < rn.j1; ++j, ++pl) {
            const int s = pl % kYS, a = pl & 1;
            ok &= ptx::mbar_wait_ff(&full[s], (pl / kYS) & 1, sAbort);
            if (pl >= 2) ok &= ptx::mbar_wait_ff(&accempty[a], ((pl >> 1) - 1) & 1, sAbort);
            ptx::tc_fence_after();
            const uint32_t bb = ptx::smem_u32(sB + (size_t)s * L::kBBytes);
            const uint32_t acc = tmem + a * kNT;
            const int bsw = 32 << rn.kc;            // B tile row bytes = its swizzle
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const uint32_t op = half ? loA : hiA;
#pragma unroll
              for (int ks = 0; ks < R / 16; ++ks) {
                if (ks >= (1 << rn.kc)) break;      // K steps past the slot's rank
                const uint64_t dOp = ptx::umma_desc_kmajor(op + ks * 32, L::kRowBytes);
                const uint64_t dB = ptx::umma_desc_kmajor(bb + ks * 32, bsw);
                ptx::tc_mma_f16(acc, swap ? dB : dOp, swap ? dOp : dB, idesc,
                                (half | ks) ? 1u : 0u);
              }
            }
            ptx::tc_commit(&accfull[a]);
          }
        }
      }
      __syncwarp();
    } else {
      // ---------------- epilogue warps 0-7
      const int q = warp & 3, h = warp >> 2;
      int pl = p, ul = u;
      for (int ri = 0; ri < n_runs; ++ri, ++ul) {
        const ExpRun rn = runs[ri];
        const int hb = ul & 1;
        const bool swap = rn.valid <= kSwapMax;
        ok &= ptx::mbar_wait_ff(&hlfull[hb], (ul >> 1) & 1, sAbort);
        const int* toks = sTok + hb * kTM;
        const float* invs = sInv + hb * kTM;
        const int m = q * 32 + lane;                  // row of this thread (normal layout)
        const int tok = toks[m];
        const float inv = invs[m];
        const int Dout = P.D_out[rn.slice];
        E* ycol = static_cast<E*>(P.y) + P.y_col_off[rn.slice];
        const int64_t ycol0 = P.y_col_off[rn.slice];
        const bool tiled = P.perm == nullptr && rn.valid == kTM;
        for (int j = rn.j0; j < rn.j1; ++j, ++pl) {
          const int s = pl % kYS, a = pl & 1;
          // a swapped pair is handled by one group of four warps (one per TMEM
          // lane quadrant), the group of its accumulator: consecutive small
          // pairs overlap; a full pair by all eight
          if (swap && a != h) continue;
          const int n0 = j * kNT, nn = min(kNT, Dout - n0);
          ok &= ptx::mbar_wait_ff(&accfull[a], (pl >> 1) & 1, sAbort);
          ok &= ptx::mbar_wait_ff(&full[s], (pl / kYS) & 1, sAbort);
          ptx::tc_fence_after();
          if (deferred >= 0) {
            // the previous TMA store of this warp's half has been read: its stage is free
            if (lane == 0) {
              ptx::bulk_wait_read_all();
              ptx::mbar_arrive(&empty[deferred]);
            }
            deferred = -1;
            __syncwarp();
          }
          char* ys = sY + (size_t)s * L::kYBytes;
          const uint32_t tacc = tmem + a * kNT + ((uint32_t)(q * 32) << 16);
          if (!swap) {
            // thread = row m, columns 64h .. 64h+63 = y half h
            if (q * 32 < rn.valid) {
              uint32_t r[64];
#pragma unroll
              for (int k = 0; k < 4; ++k) ptx::tc_ld16(tacc + 64 * h + 16 * k, r + 16 * k);
              ptx::tc_wait_ld();
              if (m < rn.valid) {
                // all eight 16-byte pieces of the row first, then the math, then
                // the stores (the loads must not wait behind earlier stores)
                char* row = ys + h * L::kYHalf + m * 128;
                uint4 w[8];
#pragma unroll
                for (int c = 0; c < 8; ++c)
                  w[c] = *reinterpret_cast<const uint4*>(row + ((c ^ (m & 7)) << 4));
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  float f[8];
                  Elem<E>::to_f32(w[c], f);
                  uint32_t o[4];
#pragma unroll
                  for (int v = 0; v < 4; ++v)
                    o[v] = Elem<E>::pack2(
                        fmaf(P.scale, __uint_as_float(r[8 * c + 2 * v]) * inv, f[2 * v]),
                        fmaf(P.scale, __uint_as_float(r[8 * c + 2 * v + 1]) * inv, f[2 * v + 1]));
                  w[c] = make_uint4(o[0], o[1], o[2], o[3]);
                }
#pragma unroll
                for (int c = 0; c < 8; ++c)
                  *reinterpret_cast<uint4*>(row + ((c ^ (m & 7)) << 4)) = w[c];
              }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&accempty[a]);
            if (tiled && nn == kNT) {
              // whole tile: one 2-D TMA store per half once its four warps are done
              ptx::fence_proxy_async_smem();
              asm volatile("bar.sync %0, 128;" ::"r"(1 + h) : "memory");
              if (q == 0) {
                if (lane == 0) {
                  ptx::tma_store_2d(&P.tmY, (int)(ycol0 + n0 + 64 * h), rn.m0,
                                    ys + h * L::kYHalf);
                  ptx::bulk_commit();
                }
                deferred = s;
              }
            } else {
              // rows 32q .. 32q+31 of half h: lane -> (row 4i + lane / 8, chunk lane % 8);
              // all shared-memory reads first, then the global stores
              const int ch = lane & 7;
              const bool col_ok = 64 * h + 8 * ch < nn;
              uint4 v[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int mr = q * 32 + 4 * i + (lane >> 3);
                v[i] = *reinterpret_cast<const uint4*>(ys + h * L::kYHalf + mr * 128 +
                                                       ((ch ^ (mr & 7)) << 4));
              }
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int lr = 4 * i + (lane >> 3);
                const int tk = __shfl_sync(0xffffffffu, tok, lr);
                if (q * 32 + lr < rn.valid && col_ok && tk >= 0)
                  *reinterpret_cast<uint4*>(ycol + (size_t)tk * P.ldy + n0 + 64 * h + 8 * ch) = v[i];
              }
              ptx::fence_proxy_async_smem();
            }
          } else {
            // swapped: thread = output column 32q + lane, all groups of 8 tokens.
            // The 8 x 8 blocks of (column, token) values are transposed across
            // the lanes 8c .. 8c+7 by shuffles, so that lane 8c + i holds token
            // 8g + i for the columns 32q + 8c .. +7: its y row piece is read
            // from the stage as 16 bytes and written straight to global memory
            // (the stage is only read, so no proxy fence before its refill).
            const int i8 = lane & 7, cb = lane >> 3;
            const int pc = (q & 1) * 4 + cb;
            const char* hbase = ys + (q >> 1) * L::kYHalf + ((pc ^ i8) << 4);
            E* ydst = ycol + n0 + q * 32 + 8 * cb;
            const bool pc_ok = q * 32 + 8 * cb < nn;
            const int ng = (rn.valid + 7) / 8;
            for (int g = 0; g < ng; ++g) {
              uint32_t r[8];
              ptx::tc_ld8(tacc + 8 * g, r);
              const int row = 8 * g + i8;            // row & 7 == i8: its swizzle phase
              const uint4 yw = *reinterpret_cast<const uint4*>(hbase + row * 128);
              const float iv = invs[row];
              const int tk = toks[row];
              ptx::tc_wait_ld();
#pragma unroll
              for (int mk = 4; mk > 0; mk >>= 1) {
                const bool up = (i8 & mk) != 0;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                  if (v & mk) continue;
                  const uint32_t got = __shfl_xor_sync(0xffffffffu, up ? r[v] : r[v | mk], mk);
                  if (up) r[v] = got;
                  else r[v | mk] = got;
                }
              }
              if (row < rn.valid && pc_ok && tk >= 0) {
                float f[8];
                Elem<E>::to_f32(yw, f);
                uint32_t o[4];
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  o[v] = Elem<E>::pack2(
                      fmaf(P.scale, __uint_as_float(r[2 * v]) * iv, f[2 * v]),
                      fmaf(P.scale, __uint_as_float(r[2 * v + 1]) * iv, f[2 * v + 1]));
                *reinterpret_cast<uint4*>(ydst + (size_t)tk * P.ldy) =
                    make_uint4(o[0], o[1], o[2], o[3]);
              }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cnt(&accempty[a], 2);   // four warps count as eight
          }
          __syncwarp();
          if (lane == 0 && deferred != s) ptx::mbar_arrive_cnt(&empty[s], swap ? 2u : 1u);
        }
        // done with this run's tokens and scales
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&hlempty[hb]);
      }
    }
    // advance the pipeline positions past this list
    for (int ri = 0; ri < n_runs; ++ri) p += runs[ri].j1 - runs[ri].j0;
    u += n_runs;
    __syncthreads();                               // the run list may be rebuilt
    lo = next_lo;
  }
  if (warp < kExpLoad0 && deferred >= 0 && lane == 0) ptx::bulk_wait_read_all();
  if (warp < kExpLoad0 && lane == 0) ptx::bulk_wait_all();
  ptx::tc_fence_before();
  __syncthreads();
  if (*sAbort) {
    // a wait timed out: let copies still in flight land before the CTA's
    // shared memory is released
    const uint64_t t0 = ptx::globaltimer_ns();
    while (ptx::globaltimer_ns() - t0 < 50000ull) {
    }
  }
  if (warp == kExpMma) ptx::tmem_dealloc(tmem, 2 * kNT);
  (void)ok;                               // every timeout also raised sAbort
  if (tid == 0 && *sAbort) atomicAdd(P.bad_meta, 1);
}

int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

template <typename E, int R>
cudaError_t shrink_tc_launch(const ShrinkArgs& a, const SegArgs& sg, lora_dtype dt,
                             cudaStream_t st, const int32_t* perm, int implicit_slots) {
  if (sg.n_seg > kMaxSegTC) return cudaErrorNotSupported;
  ShrinkTCParams P;
  memset(&P, 0, sizeof(P));
  // row gathers need a box one row high
  cudaError_t e = encode_tmap_2d(&P.tmX, dt, a.x, (uint64_t)a.D, (uint64_t)a.T,
                                 (uint64_t)a.ldx * 2, kBK, perm ? 1 : kTM, 128);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < a.n_slices; ++i) {
    e = encode_tmap_2d(&P.tmA[i], dt, a.A[i], (uint64_t)a.D, (uint64_t)a.S * R,
                       (uint64_t)a.D * 2, kBK, R, 128);
    if (e == cudaSuccess)
      e = encode_tmap_2d(&P.tmA8[i], dt, a.A[i], (uint64_t)a.D, (uint64_t)a.S * R,
                         (uint64_t)a.D * 2, kBK, 8, 128);
    if (e != cudaSuccess) return e;
  }
  const MetaHeader* hdr = reinterpret_cast<const MetaHeader*>(a.meta);
  P.meta = a.meta;
  P.seg_starts = sg.seg_starts;
  P.seg_adapter = sg.seg_adapter;
  P.n_seg = sg.n_seg;
  P.buf = a.buf;
  P.perm = perm;
  P.idx = a.idx;
  P.implicit_slots = implicit_slots;
  P.T = a.T;
  P.D = a.D;
  P.S = a.S;
  P.n_slices = a.n_slices;
  P.bad_index = const_cast<int*>(&hdr->bad_index);
  P.bad_meta = const_cast<int*>(&hdr->bad_meta);
  P.trows = implicit_slots >= kShrManySlots ? kShrRowsManySlots : kTM;
  const int max_tiles = (a.T + P.trows - 1) / P.trows + sg.n_seg;
  const int nkb_all = (a.D + kBK - 1) / kBK;
  // split K across a cluster when there are too few tiles for about 1.5 CTAs
  // per SM, each rank keeping at least 8 K blocks: up to 16 ranks (a
  // non-portable cluster size, used when the device takes it)
  const int nsm = sm_count();
  int KS = 1;
  while (KS < 16 && 2L * max_tiles * a.n_slices * KS < 3L * nsm && nkb_all >= 16 * KS) KS *= 2;
  auto kern = sgmv_shrink_tc_kernel<E, R>;
  const size_t smem = ShrinkSmem<R>::kTotal;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (KS == 16) {
    int active = 0;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(16, 1, 1);
    q.blockDim = dim3(kShrThreads, 1, 1);
    q.dynamicSmemBytes = smem;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 16;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&active, kern, &q) != cudaSuccess || active < 1) {
      cudaGetLastError();
      KS = 8;
    }
  }
  P.KS = KS;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(max_tiles * KS, a.n_slices, 1);
  cfg.blockDim = dim3(kShrThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return counted_launch(cudaLaunchKernelEx(&cfg, kern, P));
}

template <typename E, int R>
cudaError_t expand_tc_launch(const ExpandArgs& a, const SegArgs& sg, lora_dtype dt,
                             cudaStream_t st, const int32_t* perm, int implicit_slots) {
  if (sg.n_seg > kMaxSegTC) return cudaErrorNotSupported;
  ExpandTCParams P;
  memset(&P, 0, sizeof(P));
  long sum_nt = 0;
  for (int i = 0; i < a.n_slices; ++i) {
    for (int c = 0; (16 << c) <= R; ++c) {
      cudaError_t e = encode_tmap_2d(&P.tmB[c][i], dt, a.B[i], (uint64_t)R,
                                     (uint64_t)a.S * a.D_out[i], (uint64_t)R * 2, 16 << c, kNT,
                                     32 << c);
      if (e != cudaSuccess) return e;
    }
    P.y_col_off[i] = a.y_col_off[i];
    P.D_out[i] = a.D_out[i];
    sum_nt += (a.D_out[i] + kNT - 1) / kNT;
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
  P.idx = a.idx;
  P.implicit_slots = implicit_slots;
  P.T = a.T;
  P.S = a.S;
  P.n_slices = a.n_slices;
  P.scale = a.scale;
  P.bad_index = const_cast<int*>(&hdr->bad_index);
  P.bad_meta = const_cast<int*>(&hdr->bad_meta);
  P.meta = a.meta;
  P.early = a.after_shrink;
  // one CTA per SM, never more CTAs than (tile, n-tile) pairs
  const long max_tiles = (a.T + kTM - 1) / kTM + sg.n_seg;
  const long pairs = max_tiles * sum_nt;
  const int grid = (int)(pairs < sm_count() ? (pairs > 0 ? pairs : 1) : sm_count());
  auto kern = sgmv_expand_tc_kernel<E, R>;
  const size_t smem = ExpandSmem<R>::kTotal;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(exp_threads<R>(), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return counted_launch(cudaLaunchKernelEx(&cfg, kern, P));
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
