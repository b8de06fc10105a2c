// Shared device helpers and the workspace layout of liblora_b200.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lora.h"

namespace lora {

constexpr int kItemTokens = 16;     // tokens per work item of the per-token kernels
constexpr int kMaxRank = 64;

// ---------------------------------------------------------------------------
// Workspace ("meta") layout.  Offsets are multiples of 256 bytes.
//   [0, 256)       header
//   slot_off       int32 [S + 2]: slot g's tokens are perm[slot_off[g] ..
//                  slot_off[g+1]); [slot_off[S], slot_off[S+1]) = the tokens
//                  without an adapter
//   slot_rank      int32 [S]: each slot's own rank (lora_set_slot_ranks),
//                  used when the header's has_ranks is set
//   perm           int32 [T]
//   items          int4 [max_items]: {slot (-1 = none), begin, end, flags}
//   hist           int32 [group_ctas(T)][S + 1]: per-CTA slot counts of the
//                  grouping kernel
// ---------------------------------------------------------------------------
struct MetaHeader {
  int bad_index;      // count of indices outside [-1, S) (accumulates)
  int bad_meta;       // malformed segment lists, metadata built for other
                      // sizes than the call's, rows whose index disagrees
                      // with the grouping, timed-out waits (accumulates)
  int n_items;        // items in the work list
  int n_active;       // tokens with an adapter
  int T, S;           // sizes the metadata was built for
  int bar_count;      // grouping kernel's inter-CTA barrier: CTAs arrived
  int bar_gen;        //   and completed barrier generations
  int has_ranks;      // slot_rank holds per-slot ranks
  int pad[55];
};
static_assert(sizeof(MetaHeader) == 256, "header is 256 bytes");

// CTAs of the grouping kernel for T tokens: one per 512 tokens, at most 64
// (all resident at once, so they can meet at a barrier).  Measured on B200 at
// 4096 tokens: 8.8-9.3 us with 8 CTAs against 9.5 (4), 10.2-10.8 (2) and
// 9.5-10.2 us (16, 32: the barrier costs more than the split saves).
constexpr int kGroupChunkMin = 512;
constexpr int kGroupMaxCtas = 64;
__host__ __device__ inline int group_ctas(int T) {
  const int nb = (T + kGroupChunkMin - 1) / kGroupChunkMin;
  return nb < 1 ? 1 : (nb > kGroupMaxCtas ? kGroupMaxCtas : nb);
}

enum ItemFlags { kItemDirect = 1 };   // token = position (segments), no perm

struct MetaLayout {
  size_t off_slot, off_rank, off_perm, off_items, off_hist, total;
  int max_items;
  __host__ __device__ static size_t a256(size_t v) { return (v + 255) & ~size_t(255); }
  __host__ __device__ MetaLayout(int T, int S) {
    int tt = T > 0 ? T : 1;
    off_slot = 256;
    off_rank = off_slot + a256(sizeof(int) * (size_t)(S + 2));
    off_perm = off_rank + a256(sizeof(int) * (size_t)S);
    off_items = off_perm + a256(sizeof(int) * (size_t)tt);
    // per-token grouping: <= T/16 + (S + 1) items; segments: <= T/16 + n_seg
    // with n_seg <= T + 1.
    max_items = T / kItemTokens + (S + 1 > T + 1 ? S + 1 : T + 1) + 2;
    off_hist = off_items + a256(sizeof(int4) * (size_t)max_items);
    total = off_hist + a256(sizeof(int) * (size_t)group_ctas(T) * (size_t)(S + 1));
  }
};

// ---------------------------------------------------------------------------
// Element types
// ---------------------------------------------------------------------------
template <typename E> struct Elem;
template <> struct Elem<__half> {
  // 8 packed halves (16 bytes) -> 8 floats
  static __device__ __forceinline__ void to_f32(const uint4& v, float* f) {
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float2 p = __half22float2(h[k]);
      f[2 * k] = p.x;
      f[2 * k + 1] = p.y;
    }
  }
  static __device__ __forceinline__ float to_f32(uint16_t b) {
    return __half2float(__ushort_as_half(b));
  }
  static __device__ __forceinline__ uint16_t from_f32(float f) {
    return __half_as_ushort(__float2half_rn(f));
  }
  // two floats -> two packed halves (round to nearest even), a in the low half
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ void to_f32(const uint4& v, float* f) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ float to_f32(uint16_t b) {
    return __uint_as_float(((uint32_t)b) << 16);
  }
  static __device__ __forceinline__ uint16_t from_f32(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
  }
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
};

// 16-byte read-only global load (no L1 allocation for streaming data).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ldg_nc(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Work items of the metadata, or 0 (and the error counted) when the metadata
// was built for other sizes than the call's: item token positions are then not
// known to lie inside this call's buffers.
__device__ __forceinline__ int checked_items(const char* meta, int T, int S) {
  const MetaHeader* h = reinterpret_cast<const MetaHeader*>(meta);
  if (h->T == T && h->S == S) return h->n_items;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
    atomicAdd(const_cast<int*>(&h->bad_meta), 1);
  return 0;
}

// Rank slot g really uses, for a call of rank R: the slot's own rank from
// lora_set_slot_ranks rounded up to a multiple of 8, or R when none is set
// (or the value is outside (0, R)).  Rows of A and columns of B past it are
// zero padding that the kernels neither read nor multiply.
__device__ __forceinline__ int slot_rank(const char* meta, int S, int g, int R) {
  const MetaHeader* h = reinterpret_cast<const MetaHeader*>(meta);
  if (!h->has_ranks || g < 0 || g >= S) return R;
  const int v = reinterpret_cast<const int*>(meta + MetaLayout::a256(256) +
                                             MetaLayout::a256(sizeof(int) * (size_t)(S + 2)))[g];
  return (v <= 0 || v >= R) ? R : ((v + 7) & ~7);
}

// Whether token `tok` really belongs to the group of a per-token grouping it
// was placed in: idx[tok] == slot for an adapter's group, idx[tok] outside
// [0, S) for the group of tokens without an adapter.  A grouping built from
// another batch's indices (a stale workspace) fails this for every token
// whose index changed, so the kernels skip those rows and count them instead
// of computing them with the wrong adapter.
__device__ __forceinline__ bool grouped_row_ok(const int32_t* idx, int tok, int slot, int S) {
  const int v = idx[tok];
  return slot >= 0 ? v == slot : (v < 0 || v >= S);
}

__device__ __forceinline__ void count_bad_meta(const char* meta, int n) {
  atomicAdd(const_cast<int*>(&reinterpret_cast<const MetaHeader*>(meta)->bad_meta), n);
}

}  // namespace lora
