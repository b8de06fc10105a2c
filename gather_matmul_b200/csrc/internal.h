// Host-side launchers shared between the C ABI (lora_api.cu) and the kernel
// files.  Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lora.h"

namespace lora {

struct ShrinkArgs {
  const void* x;
  int64_t ldx;
  const void* A[LORA_MAX_SLICES];
  const int32_t* idx;       // per-token indices the grouping is checked against (null: segments)
  float* buf;
  int T, D, r, S, n_slices;
  const char* meta;
};

struct ExpandArgs {
  const float* buf;
  int64_t buf_slice_stride;
  const int32_t* idx;       // per-token indices the grouping is checked against (null: segments)
  const void* B[LORA_MAX_SLICES];
  int D_out[LORA_MAX_SLICES];
  int64_t y_col_off[LORA_MAX_SLICES];
  int chunk_base[LORA_MAX_SLICES + 1];   // prefix of column chunks per slice
  float scale;
  void* y;
  int64_t ldy;
  int T, r, S, n_slices;
  const char* meta;
  // 1: the kernel launched just before on the stream is this library's shrink
  // of the same batch (it writes only buf and the error counters), so the
  // tensor-core expand may read the grouping, B and y before that kernel has
  // finished and waits for it only before reading buf
  int after_shrink;
};

struct SegArgs {
  const int32_t* seg_starts;
  const int32_t* seg_adapter;
  int n_seg;
};

// Arguments of the fused per-token (BGMV) kernel: grouping, shrink and
// expand of one batch in one launch.
struct FusedArgs {
  const void* x;
  int64_t ldx;
  const void* A[LORA_MAX_SLICES];
  const void* B[LORA_MAX_SLICES];
  int D_out[LORA_MAX_SLICES];
  int64_t y_col_off[LORA_MAX_SLICES];
  void* y;
  int64_t ldy;
  float* buf;               // [n_A][T][r], n_A = shared_A ? 1 : n_slices
  const int32_t* idx;
  int* bad_index;           // meta header counters
  int* bad_meta;
  int T, D, r, S, n_slices, shared_A;
  float scale;
  int pdl_early;            // A, B and idx may be read before the previous kernel ends
};

// Every kernel launch of the library passes its status through here, so that
// lora_launch_count() reports how many launches (or stream-capture records)
// the library has made.
cudaError_t counted_launch(cudaError_t e);

// Launch attribute for programmatic dependent launch: the kernel may start
// while the previous kernel on the stream runs; every kernel of the library
// waits for its predecessor (griddepcontrol.wait) before it touches global
// memory, then lets its own successor launch.
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

cudaError_t encode_tmap_2d(CUtensorMap* map, lora_dtype dt, const void* base, uint64_t inner,
                           uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                           uint32_t box_outer, int swizzle_bytes);

// Whether the fused kernel takes this shape (host-side, no CUDA calls).
bool bgmv_fused_fits(int T, int D, int r, int n_slices, const int32_t* D_out);
// Returns cudaErrorNotSupported when the shape does not fit the fused kernel.
cudaError_t launch_bgmv_fused(lora_dtype dt, const FusedArgs& a, cudaStream_t st);

size_t group_smem_bytes(int S);
cudaError_t launch_set_ranks(int S, const int32_t* ranks, void* meta, cudaStream_t st);
// early: idx is not written by the previous launch on the stream, so the
// grouping reads and counts it before waiting for that launch (programmatic
// dependent launch) and waits only before writing the workspace
cudaError_t launch_group(int T, int S, const int32_t* idx, void* meta, cudaStream_t st,
                         int early = 0);
cudaError_t launch_segment_items(int T, int S, int n_seg, const int32_t* seg_starts,
                                 const int32_t* seg_adapter, void* meta, cudaStream_t st);

// CUDA-core kernels over the work list in meta (per-token or segment items).
cudaError_t launch_shrink_items(lora_dtype dt, const ShrinkArgs& a, int max_items,
                                cudaStream_t st);
cudaError_t launch_expand_items(lora_dtype dt, ExpandArgs a, int max_items, cudaStream_t st);

// tcgen05 tensor-core kernels for segments.  Return cudaErrorNotSupported if
// the shape has no tensor-core path (the caller then uses the item kernels).
cudaError_t launch_shrink_segment_tc(lora_dtype dt, const ShrinkArgs& a, const SegArgs& s,
                                     cudaStream_t st);
cudaError_t launch_expand_segment_tc(lora_dtype dt, const ExpandArgs& a, const SegArgs& s,
                                     cudaStream_t st);
// The same tensor-core kernels over the per-token grouping in meta (rows
// gathered through the token permutation).
cudaError_t launch_shrink_grouped_tc(lora_dtype dt, const ShrinkArgs& a, cudaStream_t st);
cudaError_t launch_expand_grouped_tc(lora_dtype dt, const ExpandArgs& a, cudaStream_t st);
// Laned shrink: all slots' A as one [S*r, D] matrix on tensor cores, each
// token's own lanes selected; needs no grouping.
cudaError_t launch_shrink_laned(lora_dtype dt, const ShrinkArgs& a, cudaStream_t st);
// Whether the per-token calls use the tensor-core kernels for this shape.
inline bool grouped_tc_preferred(int T, int r, int S) { return r >= 16 && T >= 16 * S; }

}  // namespace lora
