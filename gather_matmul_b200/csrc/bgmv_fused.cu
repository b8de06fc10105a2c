// Fused per-token (BGMV) LoRA for decode-sized batches: grouping, shrink and
// expand of one batch in ONE launch.
//
// Work decomposition.  One thread-block cluster per (adapter slot g, output
// slice i).  The CL CTAs of the cluster split the input dimension D for the
// shrink and the slice's output columns for the expand, so that each CTA
// streams 1/CL of the slot's A and B rows and of its tokens' x and y rows.
//
//   1. every CTA scans the batch's indices and keeps the tokens of slot g in
//      token order (ballot compaction), so no separate grouping launch and no
//      host round trip ("[Hardware][TPU][V1] Better tpu multilora
//      compilation": indices moved to the device; the per-token gather the
//      PyTorch baseline paid for is replaced by one read of each adapter);
//   2. the copies are issued in the order they are needed: the slot's A rows
//      (its D-chunk; fetched before the scan when the batch averages two or
//      more tokens per slot) and the first chunk's x rows feed the shrink, the
//      B rows (its output chunk, by TMA) and y rows only the expand, so the
//      shrink starts while the expand's operands are still streaming in;
//   3. per chunk of <= 16 tokens: shrink partials buf^T[r x tok] =
//      A[r x Dc] x^T[Dc x tok] run on tensor cores (mma.sync m16n8k16,
//      bf16/fp16 in, fp32 accumulate) with the tokens as the narrow n = 8
//      side, so a decode slot of 8 tokens wastes no tensor work; warps split
//      the K range and add their fragments in a fixed order; the CL partials
//      are summed in rank order through distributed shared memory, so every
//      CTA holds the full fp32 buf rows (no atomics, no pre-zeroed
//      intermediate, bitwise reproducible);
//   4. expand y[tok][o] += scale * sum_j buf[tok][j] B[o][j] on tensor cores
//      (mma.sync m16n8k16 with the tokens as M and 8 output columns as N, so
//      each thread updates adjacent column pairs of one token).  The fp32
//      intermediate enters as three half-precision terms hi + mid + lo after
//      an exact power-of-two rescale per token; the remainders are exact in
//      fp32, so the terms carry each value to about 2^-24 of the token's
//      largest one (bf16: three 8-bit significands) and the products
//      accumulate in fp32: it is never reduced to half precision ("Add
//      multi-LoRA support", Limitations list on the SGMV intermediate).  y is
//      updated in shared memory with one fp32 fma and one round-to-nearest-
//      even, then written back with coalesced 16-byte stores.
//
// Launched with programmatic dependent launch: the next kernel in the stream
// may start its own prologue while this one runs; with pdl_early the slot's
// A rows and the indices are read before waiting for the previous kernel.
// Every wait on an mbarrier is bounded; a timeout is counted in the workspace
// and the kernel finishes its cluster barriers without hanging.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace lora {

namespace {

constexpr int kFThreads = 256;
constexpr int kFWarps = kFThreads / 32;
constexpr int kTB = 16;              // tokens per chunk: two n=8 tiles
constexpr int kFusedMaxT = 4096;     // token list lives in shared memory
constexpr int kBoxRows = 256;        // TMA box height for B
constexpr size_t kMaxSmem = 227 * 1024;

struct FusedParams {
  CUtensorMap tmB[LORA_MAX_SLICES];  // B_i as [S*D_out_i rows, r cols], box {R16, 256}
  FusedArgs a;
  int CL, Dc;
};

__host__ __device__ inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Shared-memory carve-up (bytes), shared by host sizing and the kernel.
struct FusedSmem {
  int pitchA, pitchY, boxBytes, nBox;
  size_t offB, offA, offX, offY, offRed, offPart, offBuf, offTok, offCnt, offBar, total;
  __host__ __device__ FusedSmem(int R16, int Dc, int OcMax, int T, int CL) {
    pitchA = Dc * 2 + 16;
    pitchY = OcMax * 2 + 16;
    boxBytes = kBoxRows * R16 * 2;
    nBox = (OcMax + kBoxRows - 1) / kBoxRows;
    size_t o = 0;
    offB = o;  o += (size_t)boxBytes * nBox;               // 1024-aligned boxes
    offA = o;  o += (size_t)R16 * pitchA;
    offX = o;  o += (size_t)kTB * pitchA;
    offY = o;  o += (size_t)kTB * pitchY;
    o = (o + 15) & ~size_t(15);
    offRed = o;  o += sizeof(float) * kFWarps * R16 * kTB;
    offPart = o; o += sizeof(float) * CL * R16 * kTB;      // partials pushed by every rank
    offBuf = o;  o += sizeof(float) * R16 * kTB;
    offTok = o;  o += sizeof(int) * (size_t)(T > 0 ? T : 1);
    offCnt = o;  o += sizeof(int) * (kFWarps + 1);
    o = (o + 7) & ~size_t(7);
    offBar = o;  o += 4 * sizeof(uint64_t);
    total = o + 1024;                                      // base alignment slack
  }
};

template <int R16>
__device__ __forceinline__ int swz_chunk(int row, int chunk) {
  // TMA 32/64/128-byte swizzle: the 16-byte chunk index is XORed with bits of
  // the row's position inside the 256/512/1024-byte swizzle atom.
  if constexpr (R16 == 64) return chunk ^ (row & 7);
  else if constexpr (R16 == 32) return chunk ^ ((row >> 1) & 3);
  else return chunk ^ ((row >> 2) & 1);
}

template <typename E, int R16>
__global__ void __launch_bounds__(kFThreads, 2)
bgmv_fused_kernel(const __grid_constant__ FusedParams P) {
  constexpr bool kBF = std::is_same<E, __nv_bfloat16>::value;
  constexpr int MT = R16 / 16;
  const FusedArgs& a = P.a;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = P.CL;
  const int crank = (int)cluster.block_rank();
  const int unit = blockIdx.x / CL;
  const int g = unit % a.S;
  const int slice = unit / a.S;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = a.r;

  int oc_max = 0;
  for (int i = 0; i < a.n_slices; ++i)
    oc_max = max(oc_max, round_up((a.D_out[i] + CL - 1) / CL, 16));
  const FusedSmem L(R16, P.Dc, oc_max, a.T, CL);
  extern __shared__ char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  char* sB = smem + L.offB;
  char* sA = smem + L.offA;
  char* sX = smem + L.offX;
  char* sY = smem + L.offY;
  float* sRed = reinterpret_cast<float*>(smem + L.offRed);
  float* sRecv = reinterpret_cast<float*>(smem + L.offPart);
  float* sBuf = reinterpret_cast<float*>(smem + L.offBuf);
  int* sTok = reinterpret_cast<int*>(smem + L.offTok);
  int* sCnt = reinterpret_cast<int*>(smem + L.offCnt);
  uint64_t* barA = reinterpret_cast<uint64_t*>(smem + L.offBar);   // A rows (once)
  uint64_t* barB = barA + 1;                                          // B tiles (once)
  uint64_t* barX = barA + 2;                                          // x rows (per chunk)
  uint64_t* barY = barA + 3;                                          // y rows (per chunk)

  const int D = a.D;
  const int d0 = crank * P.Dc;
  const int dn = max(0, min(D, d0 + P.Dc) - d0);           // this CTA's shrink columns
  const int Dout = a.D_out[slice];
  const int Oc = round_up((Dout + CL - 1) / CL, 16);
  const int o0 = crank * Oc;
  const int on = max(0, min(Dout, o0 + Oc) - o0);          // this CTA's output columns
  const int aslice = a.shared_A ? 0 : slice;
  const E* Ag = static_cast<const E*>(a.A[aslice]) + (size_t)g * R * D + d0;
  const E* x = static_cast<const E*>(a.x);
  E* y = static_cast<E*>(a.y);
  const int64_t yoff = a.y_col_off[slice] + o0;

  if (tid == 0) {
    ptx::mbar_init(barA, kFWarps);   // one expect_tx arrival per issuing warp
    ptx::mbar_init(barB, kFWarps);
    ptx::mbar_init(barX, kFWarps);
    ptx::mbar_init(barY, kFWarps);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&P.tmB[slice]);
  }
  // zero the k tail [dn, round16(dn)) of the A and x tiles so a partial last
  // k-step multiplies zeros, and the unused rank rows of a padded A tile
  {
    const int kpad = round_up(dn, 16) - dn;   // 0 or 8 columns
    if (kpad)
      for (int rr = tid; rr < R16 + kTB; rr += kFThreads) {
        char* row = rr < R16 ? sA + (size_t)rr * L.pitchA : sX + (size_t)(rr - R16) * L.pitchA;
        *reinterpret_cast<uint4*>(row + dn * 2) = make_uint4(0, 0, 0, 0);
      }
    for (int e = tid; e < (R16 - R) * (L.pitchA / 16); e += kFThreads)
      reinterpret_cast<uint4*>(sA + (size_t)R * L.pitchA)[e] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();

  // Copies are issued in the order they are needed: the slot's A rows and the
  // first chunk's x rows feed the shrink, B and y only the expand.  When the
  // batch has at least two tokens per slot on average the slot's A rows and B
  // tiles (they depend on the slot alone) are fetched before the index scan,
  // on the guess that this slot has tokens; a CTA whose slot turns out empty
  // waits for them before it exits.
  const bool spec_A = a.T >= 2 * a.S;
  auto issue_A = [&]() {
    if (lane == 0) {
      const int nA = dn > 0 ? (R - warp + kFWarps - 1) / kFWarps : 0;   // rows warp, warp+8, ..
      ptx::mbar_arrive_expect_tx(barA, (uint32_t)(max(nA, 0) * dn * 2));
      if (dn > 0)
        for (int j = warp; j < R; j += kFWarps)
          ptx::bulk_g2s(sA + (size_t)j * L.pitchA, Ag + (size_t)j * D, dn * 2, barA);
    }
  };
  auto issue_B = [&]() {
    if (lane == 0) {
      const int nbox = (on + kBoxRows - 1) / kBoxRows;
      const int nB = (nbox - warp + kFWarps - 1) / kFWarps;
      ptx::mbar_arrive_expect_tx(barB, (uint32_t)(max(nB, 0) * L.boxBytes));
      for (int b = warp; b < nbox; b += kFWarps)
        ptx::tma_load_2d(sB + (size_t)b * L.boxBytes, &P.tmB[slice], 0,
                         g * Dout + o0 + b * kBoxRows, barB);
    }
  };
  if (!a.pdl_early) ptx::grid_dep_wait();
  // the first block of indices is requested ahead of the A rows, so that the
  // scan does not queue behind them; each block prefetches the next
  int v_next = tid < a.T ? a.idx[tid] : -1;
  if (spec_A) {
    issue_A();
    issue_B();
  }

  // 1. this slot's tokens, in token order
  int n_tok = 0;
  int bad = 0;
  const bool counter = (unit == 0 && crank == 0);
  for (int base = 0; base < a.T; base += kFThreads) {
    const int t = base + tid;
    const int v = v_next;
    if (base + kFThreads < a.T) v_next = t + kFThreads < a.T ? a.idx[t + kFThreads] : -1;
    if (counter && t < a.T && (v < -1 || v >= a.S)) ++bad;
    const bool hit = (v == g);
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) sCnt[warp] = __popc(bal);
    __syncthreads();
    int pre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) {
      const int c = sCnt[w];
      pre += w < warp ? c : 0;
      tot += c;
    }
    if (hit) sTok[n_tok + pre + __popc(bal & lanemask_lt())] = t;
    n_tok += tot;
    __syncthreads();
  }
  if (counter) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
    if (lane == 0 && bad) atomicAdd(a.bad_index, bad);
  }
  if (counter && a.buf != nullptr) {
    // tokens without an adapter get zero buf rows; buf may still be read by
    // the previous kernel, so this waits for it first
    if (a.pdl_early) ptx::grid_dep_wait();
    const int na = a.shared_A ? 1 : a.n_slices;
    for (int e = tid; e < a.T * R; e += kFThreads) {
      const int t = e / R;
      const int v = a.idx[t];
      if (v < 0 || v >= a.S)
        for (int i = 0; i < na; ++i) a.buf[((size_t)i * a.T + t) * R + e % R] = 0.f;
    }
  }
  ptx::grid_dep_launch_dependents();
  if (n_tok == 0) {                 // the same for every CTA of the cluster
    if (spec_A && tid == 0) {         // the A rows and B tiles fetched on a guess
      ptx::mbar_wait(barA, 0);
      ptx::mbar_wait(barB, 0);
    }
    return;
  }

  bool ok = true;
  if (!spec_A) issue_A();
  if (a.pdl_early) ptx::grid_dep_wait();
  // x and y row chunks of tokens c0 .. c0+nt-1 (token k by warp k % 8)
  auto issue_x = [&](int c0, int nt) {
    if (lane == 0) {
      const int nk = max((nt - warp + kFWarps - 1) / kFWarps, 0);
      ptx::mbar_arrive_expect_tx(barX, (uint32_t)(nk * dn * 2));
      if (dn > 0)
        for (int k = warp; k < nt; k += kFWarps)
          ptx::bulk_g2s(sX + (size_t)k * L.pitchA, x + (size_t)sTok[c0 + k] * a.ldx + d0, dn * 2,
                        barX);
    }
  };
  auto issue_y = [&](int c0, int nt) {
    if (lane == 0) {
      const int nk = max((nt - warp + kFWarps - 1) / kFWarps, 0);
      ptx::mbar_arrive_expect_tx(barY, (uint32_t)(nk * on * 2));
      if (on > 0)
        for (int k = warp; k < nt; k += kFWarps)
          ptx::bulk_g2s(sY + (size_t)k * L.pitchY, y + (size_t)sTok[c0 + k] * a.ldy + yoff, on * 2,
                        barY);
    }
  };
  // 2. the first chunk's x rows, the slot's B rows (output chunk), the first
  // chunk's y rows; lane 0 of every warp issues its share
  issue_x(0, min(kTB, n_tok));
  if (!spec_A) issue_B();
  issue_y(0, min(kTB, n_tok));

  int phase = 0;
  for (int c0 = 0; c0 < n_tok; c0 += kTB, phase ^= 1) {
    const int nt = min(kTB, n_tok - c0);
    const int NT = nt > 8 ? 2 : 1;
    // 3a. this chunk's x and y row chunks (the first chunk's are on their way)
    if (c0 > 0) {
      issue_x(c0, nt);
      issue_y(c0, nt);
    }
    if (c0 == 0) ok &= ptx::mbar_wait(barA, 0);
    ok &= ptx::mbar_wait(barX, phase);

    // 3b. shrink partial over this CTA's columns: warps split the k-steps
    {
      float acc[MT][2][4];
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[m][n][q] = 0.f;
      const int KS = (dn + 15) / 16;
      const uint32_t aBase = ptx::smem_u32(sA) + (lane & 15) * L.pitchA + (lane >> 4) * 16;
      const uint32_t xBase =
          ptx::smem_u32(sX) + ((lane & 7) + 8 * (lane >> 4)) * L.pitchA + ((lane >> 3) & 1) * 16;
      for (int ks = warp; ks < KS; ks += kFWarps) {
        uint32_t xb[4];
        ptx::ldsm_x4(xBase + ks * 32, xb[0], xb[1], xb[2], xb[3]);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          uint32_t af[4];
          ptx::ldsm_x4(aBase + m * 16 * L.pitchA + ks * 32, af[0], af[1], af[2], af[3]);
          ptx::mma_16816<kBF>(acc[m][0], af, xb[0], xb[1]);
          if (NT == 2) ptx::mma_16816<kBF>(acc[m][1], af, xb[2], xb[3]);
        }
      }
      // fragment -> sRed[warp][j][t]
      float* red = sRed + warp * R16 * kTB;
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const int j = m * 16 + (lane >> 2);
          const int t = n * 8 + 2 * (lane & 3);
          red[j * kTB + t] = acc[m][n][0];
          red[j * kTB + t + 1] = acc[m][n][1];
          red[(j + 8) * kTB + t] = acc[m][n][2];
          red[(j + 8) * kTB + t + 1] = acc[m][n][3];
        }
    }
    // peers must be done reading their receive buffers of the previous chunk
    if (c0 > 0) cluster.sync();
    else __syncthreads();
    // CTA partial, pushed into slot [crank] of every rank's receive buffer
    for (int e = tid * 4; e < R16 * kTB; e += kFThreads * 4) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kFWarps; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(sRed + w * R16 * kTB + e);
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
      }
      for (int q = 0; q < CL; ++q)
        *reinterpret_cast<float4*>(cluster.map_shared_rank(sRecv, q) + crank * R16 * kTB + e) = s;
    }
    cluster.sync();                       // every rank's partial has arrived
    for (int e = tid; e < R16 * kTB; e += kFThreads) {
      float s = 0.f;
      for (int q = 0; q < CL; ++q) s += sRecv[q * R16 * kTB + e];
      const int k = e % kTB, j = e / kTB;   // full sum over D, same in every CTA
      sBuf[k * R16 + j] = s;
    }
    __syncthreads();

    // 3c. the intermediate: stored once per cluster
    if (a.buf != nullptr && crank == 0 && (slice == 0 || !a.shared_A)) {
      float* bo = a.buf + (size_t)aslice * a.T * R;
      for (int e = tid; e < nt * R; e += kFThreads) {
        const int k = e / R, j = e % R;
        bo[(size_t)sTok[c0 + k] * R + j] = sBuf[k * R16 + j];
      }
    }

    // 3d. expand on tensor cores: y[t][o] += scale * sum_j buf[t][j] B[o][j]
    // with mma.sync m16n8k16 (M = 16 token rows, N = 8 output columns,
    // K = 16), so each thread's results are pairs of adjacent columns of one
    // token: 32-bit y updates.  The fp32 intermediate enters as three
    // bf16/fp16 terms hi + mid + lo after an exact power-of-two rescale per
    // token: hi is buf rounded, mid the rounded remainder, lo the rounded
    // remainder of that; both remainders are exact in fp32, so the terms carry
    // the full fp32 value (bf16: 3 x 8 significant bits) and the products
    // accumulate in fp32.
    {
      constexpr int PH = R16 * 2 + 16;                // operand row pitch (bytes)
      char* sH = reinterpret_cast<char*>(sRed);       // [3][kTB][PH]; sRed is free here
      float* sInvT = reinterpret_cast<float*>(sH + 3 * kTB * PH);
      {
        const int k = 2 * warp + (lane >> 4), li = lane & 15;   // token k, lanes of a half
        constexpr int JL = R16 / 16;
        float v[JL];
        float mx = 0.f;
#pragma unroll
        for (int u = 0; u < JL; ++u) {
          v[u] = k < nt ? sBuf[k * R16 + li + 16 * u] : 0.f;
          mx = fmaxf(mx, fabsf(v[u]));
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int ex = ((__float_as_int(mx) >> 23) & 0xff) - 127;
        ex = (mx > 0.f && ex > -100 && ex < 100) ? ex : 0;
        const float sc = __int_as_float((127 - ex + 7) << 23);
        if (li == 0) sInvT[k] = __int_as_float((127 + ex - 7) << 23);
#pragma unroll
        for (int u = 0; u < JL; ++u) {
          const float w0 = v[u] * sc;
          const uint16_t h0 = Elem<E>::from_f32(w0);
          const float w1 = w0 - Elem<E>::to_f32(h0);
          const uint16_t h1 = Elem<E>::from_f32(w1);
          const uint16_t h2 = Elem<E>::from_f32(w1 - Elem<E>::to_f32(h1));
          char* row = sH + k * PH + (li + 16 * u) * 2;
          *reinterpret_cast<uint16_t*>(row) = h0;
          *reinterpret_cast<uint16_t*>(row + kTB * PH) = h1;
          *reinterpret_cast<uint16_t*>(row + 2 * kTB * PH) = h2;
        }
      }
      if (c0 == 0) ok &= ptx::mbar_wait(barB, 0);
      ok &= ptx::mbar_wait(barY, phase);
      __syncthreads();
      // A fragments (token rows) of the three terms; B fragments: output rows
      const uint32_t aBase = ptx::smem_u32(sH) + (lane & 15) * PH + (lane >> 4) * 16;
      const int t0 = lane >> 2;                        // this thread's token rows t0, t0 + 8
      const float inv0 = sInvT[t0], inv1 = sInvT[t0 + 8];
      char* yrow0 = sY + (size_t)t0 * L.pitchY + 4 * (lane & 3);
      char* yrow1 = yrow0 + 8 * (size_t)L.pitchY;
      const bool row0 = t0 < nt, row1 = NT == 2 && t0 + 8 < nt;
      const int MTo = (on + 15) / 16;
#pragma unroll 1
      for (int mt = warp; mt < MTo; mt += kFWarps) {
        float acc[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[n][q] = 0.f;
        // B rows mt*16 + 0..15: lanes 0-15 the first 8 rows (k chunks 0/1),
        // lanes 16-31 the next 8
        const int orow = mt * 16 + (lane & 7) + 8 * (lane >> 4);
        const char* brow = sB + (size_t)(orow / kBoxRows) * L.boxBytes +
                           (size_t)(orow % kBoxRows) * (R16 * 2);
#pragma unroll
        for (int ks = 0; ks < R16 / 16; ++ks) {
          uint32_t bf[4];
          ptx::ldsm_x4(ptx::smem_u32(brow + swz_chunk<R16>(orow % kBoxRows,
                                                           2 * ks + ((lane >> 3) & 1)) * 16),
                       bf[0], bf[1], bf[2], bf[3]);
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            uint32_t af[4];
            ptx::ldsm_x4(aBase + term * kTB * PH + ks * 32, af[0], af[1], af[2], af[3]);
            ptx::mma_16816<kBF>(acc[0], af, bf[0], bf[1]);
            ptx::mma_16816<kBF>(acc[1], af, bf[2], bf[3]);
          }
        }
        // acc[n][0..1]: token t0, columns o, o+1 with o = 16 mt + 8n + 2 (lane%4);
        // acc[n][2..3]: token t0 + 8
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const int o = mt * 16 + 8 * n + 2 * (lane & 3);
          if (o < on) {                               // on is a multiple of 8
            uint32_t* p0 = reinterpret_cast<uint32_t*>(yrow0 + (mt * 16 + 8 * n) * 2);
            uint32_t* p1 = reinterpret_cast<uint32_t*>(yrow1 + (mt * 16 + 8 * n) * 2);
            const uint32_t w0 = row0 ? *p0 : 0u;
            const uint32_t w1 = row1 ? *p1 : 0u;
            const uint16_t* h0 = reinterpret_cast<const uint16_t*>(&w0);
            const uint16_t* h1 = reinterpret_cast<const uint16_t*>(&w1);
            if (row0)
              *p0 = Elem<E>::pack2(fmaf(a.scale, acc[n][0] * inv0, Elem<E>::to_f32(h0[0])),
                                   fmaf(a.scale, acc[n][1] * inv0, Elem<E>::to_f32(h0[1])));
            if (row1)
              *p1 = Elem<E>::pack2(fmaf(a.scale, acc[n][2] * inv1, Elem<E>::to_f32(h1[0])),
                                   fmaf(a.scale, acc[n][3] * inv1, Elem<E>::to_f32(h1[1])));
          }
        }
      }
    }
    __syncthreads();
    // 3e. coalesced 16-byte stores of the updated y row chunks
    {
      const int cpr = on / 8;                  // 16-byte chunks per row
      for (int e = tid; e < nt * cpr; e += kFThreads) {
        const int k = e / cpr, c = e % cpr;
        *reinterpret_cast<uint4*>(y + (size_t)sTok[c0 + k] * a.ldy + yoff + c * 8) =
            *reinterpret_cast<const uint4*>(sY + (size_t)k * L.pitchY + c * 16);
      }
    }
    if (c0 + kTB < n_tok) {
      // the next chunk's copies (async proxy) overwrite sX / sY that this
      // chunk read and wrote through the generic proxy
      ptx::fence_proxy_async_smem();
      __syncthreads();
    }
  }
  if (!ok && tid == 0) atomicAdd(a.bad_meta, 1);
}

// Cluster size and per-CTA chunks for a shape and a cluster size.
struct FusedPlan {
  int CL, Dc, oc_max, R16;
  size_t smem;
};

FusedPlan fused_plan(int T, int D, int r, int n_slices, const int32_t* D_out, int CL) {
  FusedPlan p;
  p.R16 = r < 16 ? 16 : r;
  p.CL = CL;
  p.Dc = round_up((D + CL - 1) / CL, 16);
  p.oc_max = 0;
  for (int i = 0; i < n_slices; ++i) {
    int oc = round_up((D_out[i] + CL - 1) / CL, 16);
    p.oc_max = p.oc_max > oc ? p.oc_max : oc;
  }
  p.smem = FusedSmem(p.R16, p.Dc, p.oc_max, T, CL).total;
  return p;
}

constexpr int kClusterSizes[4] = {8, 4, 2, 1};

template <typename E, int R16>
cudaError_t fused_launch(const FusedArgs& a, lora_dtype dt, cudaStream_t st) {
  auto kern = bgmv_fused_kernel<E, R16>;
  const int units = a.S * a.n_slices;
  // Largest cluster size whose whole grid is co-resident (one wave); the
  // partial-sum exchange then never waits on a cluster that has not started.
  FusedPlan plan;
  plan.CL = 0;
  FusedPlan fallback;
  fallback.CL = 0;
  for (int CL : kClusterSizes) {
    FusedPlan p = fused_plan(a.T, a.D, a.r, a.n_slices, a.D_out, CL);
    if (p.smem > kMaxSmem) continue;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(units * CL, 1, 1);
    q.blockDim = dim3(kFThreads, 1, 1);
    q.dynamicSmemBytes = p.smem;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = CL;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kern, &q) != cudaSuccess) {
      cudaGetLastError();
      active = 0;
    }
    if (fallback.CL == 0 && active > 0) fallback = p;
    if (active >= units) {
      plan = p;
      break;
    }
  }
  if (plan.CL == 0) plan = fallback;
  if (plan.CL == 0) return cudaErrorNotSupported;

  FusedParams P;
  memset(&P, 0, sizeof(P));
  P.a = a;
  P.CL = plan.CL;
  P.Dc = plan.Dc;
  for (int i = 0; i < a.n_slices; ++i) {
    cudaError_t e = encode_tmap_2d(&P.tmB[i], dt, a.B[i], (uint64_t)a.r,
                                   (uint64_t)a.S * a.D_out[i], (uint64_t)a.r * 2, R16, kBoxRows,
                                   R16 * 2);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(units * plan.CL, 1, 1);
  cfg.blockDim = dim3(kFThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return counted_launch(cudaLaunchKernelEx(&cfg, kern, P));
}

}  // namespace

bool bgmv_fused_fits(int T, int D, int r, int n_slices, const int32_t* D_out) {
  if (T > kFusedMaxT) return false;
  for (int CL : kClusterSizes)
    if (fused_plan(T, D, r, n_slices, D_out, CL).smem <= kMaxSmem) return true;
  return false;
}

cudaError_t launch_bgmv_fused(lora_dtype dt, const FusedArgs& a, cudaStream_t st) {
  if (!bgmv_fused_fits(a.T, a.D, a.r, a.n_slices, a.D_out)) return cudaErrorNotSupported;
  switch (a.r < 16 ? 16 : a.r) {
    case 16: return dt == LORA_BF16 ? fused_launch<__nv_bfloat16, 16>(a, dt, st)
                                    : fused_launch<__half, 16>(a, dt, st);
    case 32: return dt == LORA_BF16 ? fused_launch<__nv_bfloat16, 32>(a, dt, st)
                                    : fused_launch<__half, 32>(a, dt, st);
    case 64: return dt == LORA_BF16 ? fused_launch<__nv_bfloat16, 64>(a, dt, st)
                                    : fused_launch<__half, 64>(a, dt, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace lora
