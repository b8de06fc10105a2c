// Laned shrink: every slot's adapter in one dense tensor-core contraction,
// then each token keeps its own slot's lanes.  No grouping, no sort.
//
// "[Hardware][TPU][V1] Better tpu multilora compilation" describes the TPU
// kernels' LoRA laning: several adapters packed side by side in one vector
// register, so that one pass serves tokens of different adapters.  The sm_100a
// analogue here treats the slot-major stack A_i [S, r, D] as one matrix of
// S*r rows ("lanes") and computes
//   C[t][l] = sum_d x[t][d] * A_i[l / r][l % r][d]      for all lanes l,
// a dense M = tokens x N = S*r x K = D contraction on tcgen05 (TMA 2-D tiles,
// fp32 accumulator in tensor memory), then
//   buf[i][t][j] = C[t][idx[t] * r + j]
// read straight out of tensor memory.  The contraction does S times the
// useful multiply-adds, but for small ranks that work sits far below the
// tensor-core roofline (cfg. decode: 256 tokens x 512 lanes x 4096), while
// every byte is read once, in dense tiles, without the index scan, the
// permutation and the row gathers of the grouped path.
//
// Work decomposition: one CTA per (128-token tile, 128-lane tile, K range);
// the KS CTAs of one (token, lane) tile form a cluster that splits K and adds
// the selected lanes of its partial sums in rank order through distributed
// shared memory.  Lanes of one slot never straddle two lane tiles (128 is a
// multiple of every supported rank), so each token's buf row is written by
// exactly one lane tile; rows of tokens without an adapter are written as
// zeros by lane tile 0.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace lora {

namespace {

constexpr int kLM = 128;      // tokens per tile (MMA M)
constexpr int kLN = 128;      // lanes per tile (MMA N)
constexpr int kLK = 64;       // K per stage: one 128-byte swizzled row
constexpr int kLStages = 3;
constexpr int kLThreads = 160;   // warps 0-3: loads, then epilogue; warp 4: MMA

struct LanedSmem {
  static constexpr int kXBytes = kLM * 128;
  static constexpr int kABytes = kLN * 128;
  static constexpr int kStageBytes = kXBytes + kABytes;
  static constexpr size_t kBar = (size_t)kStageBytes * kLStages;
  static constexpr size_t kTotal = kBar + 8 * (2 * kLStages + 1) + 64 + 1024;
};
static_assert(2 * (LanedSmem::kTotal + 1024) <= 228 * 1024, "two laned CTAs per SM");

struct LanedParams {
  CUtensorMap tmX;                       // x as [T rows, D cols], box {64, 128}
  CUtensorMap tmA[LORA_MAX_SLICES];      // A_i as [S*r rows, D cols], box {64, 128}
  const int32_t* idx;
  float* buf;
  int* bad_index;
  int* bad_meta;
  int T, D, S, n_slices, KS, n_lane_tiles;
};

template <typename E, int R>
__global__ void __launch_bounds__(kLThreads, 2)
laned_shrink_kernel(const __grid_constant__ LanedParams P) {
  using L = LanedSmem;
  constexpr bool kBF = std::is_same<E, __nv_bfloat16>::value;
  constexpr uint32_t kIdesc = ptx::umma_idesc_f16(kBF, kLM, kLN);
  constexpr int kPitch = R + 4;                       // floats, received partial rows
  ptx::grid_dep_wait();               // x, A and idx producers have finished
  ptx::grid_dep_launch_dependents();
  cg::cluster_group cluster = cg::this_cluster();
  const int KS = P.KS;
  const int kr = (int)cluster.block_rank();
  const int unit = blockIdx.x / KS;
  const int lt = unit % P.n_lane_tiles;               // lane tile
  const int mt = unit / P.n_lane_tiles;               // token tile
  const int m0 = mt * kLM, n0 = lt * kLN;
  const int slice = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + kLStages;
  uint64_t* accbar = empty + kLStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accbar + 1);

  const int nkb_all = (P.D + kLK - 1) / kLK;
  const int kb0 = kr * nkb_all / KS, kb1 = (kr + 1) * nkb_all / KS;
  const int nkb = kb1 - kb0;                          // >= 1 (the host keeps KS <= nkb_all)

  if (tid == 0) {
    for (int s = 0; s < kLStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accbar, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&P.tmX);
    ptx::prefetch_tensormap(&P.tmA[slice]);
  }
  if (warp == 4) {
    ptx::tmem_alloc(tmem_slot, kLN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  if (warp == 0 && lane == 0) {
    // loads: the token tile and the lane tile of each K block
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kLStages;
      if (i >= kLStages) ok &= ptx::mbar_wait(&empty[s], ((i / kLStages) - 1) & 1);
      char* st = smem + (size_t)s * L::kStageBytes;
      const int kx = (kb0 + i) * kLK;
      ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)L::kStageBytes);
      ptx::tma_load_2d(st, &P.tmX, kx, m0, &full[s]);
      ptx::tma_load_2d(st + L::kXBytes, &P.tmA[slice], kx, n0, &full[s]);
    }
  } else if (warp == 4 && lane == 0) {
    const uint32_t sbase = ptx::smem_u32(smem);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kLStages;
      ok &= ptx::mbar_wait(&full[s], (i / kLStages) & 1);
      ptx::tc_fence_after();
      const uint32_t xa = sbase + s * L::kStageBytes, aa = xa + L::kXBytes;
#pragma unroll
      for (int k = 0; k < kLK / 16; ++k)
        ptx::tc_mma_f16(tmem, ptx::umma_desc_kmajor(xa + k * 32, 128),
                        ptx::umma_desc_kmajor(aa + k * 32, 128), kIdesc,
                        (i > 0 || k > 0) ? 1u : 0u);
      ptx::tc_commit(&empty[s]);
    }
    ptx::tc_commit(accbar);
  }
  __syncwarp();
  ok &= ptx::mbar_wait(accbar, 0);
  ptx::tc_fence_after();

  // epilogue: thread = token row m (warps 0-3, TMEM lane quadrant = warp);
  // keep the R lanes of the token's own slot when they lie in this lane tile
  const bool has_row = warp < 4;
  const int m = warp * 32 + lane;
  const int t = m0 + m;
  int g = -1;
  if (has_row && t < P.T) {
    g = P.idx[t];
    if (g < -1 || g >= P.S) {
      if (lt == 0 && kr == 0 && slice == 0) atomicAdd(P.bad_index, 1);
      g = -1;
    }
  }
  const int lane0 = g >= 0 ? g * R - n0 : -1;
  const bool mine = lane0 >= 0 && lane0 < kLN;
  float v[R];
#pragma unroll
  for (int u = 0; u < R; ++u) v[u] = 0.f;
  if (has_row) {
#pragma unroll
    for (int b = 0; b < kLN / R; ++b) {
      if constexpr (R == 8) {
        uint32_t r8[8];
        ptx::tc_ld8(tmem + ((uint32_t)(warp * 32) << 16) + b * 8, r8);
        ptx::tc_wait_ld();
        if (lane0 == b * 8) {
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = __uint_as_float(r8[u]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < R / 16; ++c) {
          uint32_t r16[16];
          ptx::tc_ld16(tmem + ((uint32_t)(warp * 32) << 16) + b * R + c * 16, r16);
          ptx::tc_wait_ld();
          if (lane0 == b * R) {
#pragma unroll
            for (int u = 0; u < 16; ++u) v[c * 16 + u] = __uint_as_float(r16[u]);
          }
        }
      }
    }
  }
  float* bufs = P.buf + (size_t)slice * P.T * R;
  // tokens without an adapter: zero rows, from lane tile 0's rank 0
  const bool zero_row = has_row && t < P.T && g < 0 && lt == 0 && kr == 0;
  if (zero_row) {
    float4* row = reinterpret_cast<float4*>(bufs + (size_t)t * R);
#pragma unroll
    for (int q = 0; q < R / 4; ++q) row[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (KS == 1) {
    if (mine && t < P.T) {
      float4* row = reinterpret_cast<float4*>(bufs + (size_t)t * R);
#pragma unroll
      for (int q = 0; q < R / 4; ++q)
        row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  } else {
    // row m is owned by rank m / rows; every rank pushes its partial of the
    // row into slot [kr] of the owner's receive area (its drained stages),
    // then each owner adds its KS slots in rank order
    const int rows = kLM / KS;
    cluster.barrier_arrive();                 // this CTA's MMAs and stages are done...
    cluster.barrier_wait();                   // ...and so are every peer's
    float* recv = reinterpret_cast<float*>(smem);
    if (mine) {
      float* dst = cluster.map_shared_rank(recv, m / rows) + (size_t)(kr * rows + m % rows) * kPitch;
#pragma unroll
      for (int q = 0; q < R / 4; ++q)
        reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
    cluster.sync();                           // every partial has arrived
    for (int e = tid; e < rows * R; e += kLThreads) {
      const int lm = e / R, j = e % R;
      const int tt = m0 + kr * rows + lm;
      if (tt >= P.T) continue;
      const int gg = P.idx[tt];
      if (gg < 0 || gg >= P.S || gg * R - n0 < 0 || gg * R - n0 >= kLN) continue;
      float sum = 0.f;
      for (int q = 0; q < KS; ++q) sum += recv[(size_t)(q * rows + lm) * kPitch + j];
      bufs[(size_t)tt * R + j] = sum;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 4) ptx::tmem_dealloc(tmem, kLN);
  if (!ok && tid == 0) atomicAdd(P.bad_meta, 1);
}

int sm_count_laned() {
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
cudaError_t laned_launch(const ShrinkArgs& a, lora_dtype dt, cudaStream_t st) {
  LanedParams P;
  memset(&P, 0, sizeof(P));
  cudaError_t e = encode_tmap_2d(&P.tmX, dt, a.x, (uint64_t)a.D, (uint64_t)a.T,
                                 (uint64_t)a.ldx * 2, kLK, kLM, 128);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < a.n_slices; ++i) {
    e = encode_tmap_2d(&P.tmA[i], dt, a.A[i], (uint64_t)a.D, (uint64_t)a.S * R,
                       (uint64_t)a.D * 2, kLK, kLN, 128);
    if (e != cudaSuccess) return e;
  }
  const MetaHeader* hdr = reinterpret_cast<const MetaHeader*>(a.meta);
  P.idx = a.idx;
  P.buf = a.buf;
  P.bad_index = const_cast<int*>(&hdr->bad_index);
  P.bad_meta = const_cast<int*>(&hdr->bad_meta);
  P.T = a.T;
  P.D = a.D;
  P.S = a.S;
  P.n_slices = a.n_slices;
  const int m_tiles = (a.T + kLM - 1) / kLM;
  P.n_lane_tiles = (a.S * R + kLN - 1) / kLN;
  const int units = m_tiles * P.n_lane_tiles * a.n_slices;
  const int nkb_all = (a.D + kLK - 1) / kLK;
  // split K over a cluster until the grid fills about two CTAs per SM, each
  // rank keeping at least two K blocks: up to 16 ranks (non-portable size,
  // used when the device takes it)
  const int nsm = sm_count_laned();
  int KS = 1;
  while (KS < 16 && units * KS * 2 <= 2 * nsm && nkb_all >= 4 * KS) KS *= 2;
  auto kern = laned_shrink_kernel<E, R>;
  const size_t smem = LanedSmem::kTotal;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (KS == 16) {
    int active = 0;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(16, 1, 1);
    q.blockDim = dim3(kLThreads, 1, 1);
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
  cfg.gridDim = dim3(m_tiles * P.n_lane_tiles * KS, a.n_slices, 1);
  cfg.blockDim = dim3(kLThreads, 1, 1);
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

}  // namespace

cudaError_t launch_shrink_laned(lora_dtype dt, const ShrinkArgs& a, cudaStream_t st) {
  if (a.D % 8 != 0 || a.ldx % 8 != 0) return cudaErrorNotSupported;
  const bool bf = dt == LORA_BF16;
  switch (a.r) {
    case 8: return bf ? laned_launch<__nv_bfloat16, 8>(a, dt, st) : laned_launch<__half, 8>(a, dt, st);
    case 16: return bf ? laned_launch<__nv_bfloat16, 16>(a, dt, st) : laned_launch<__half, 16>(a, dt, st);
    case 32: return bf ? laned_launch<__nv_bfloat16, 32>(a, dt, st) : laned_launch<__half, 32>(a, dt, st);
    case 64: return bf ? laned_launch<__nv_bfloat16, 64>(a, dt, st) : laned_launch<__half, 64>(a, dt, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace lora
