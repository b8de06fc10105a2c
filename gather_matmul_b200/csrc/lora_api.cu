// extern "C" entry points of liblora_b200.so: host-side argument checks and
// dispatch to the kernels.  See include/lora.h for the contract of each call.
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

using namespace lora;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool rank_ok(int r) { return r == 8 || r == 16 || r == 32 || r == 64; }

lora_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA; }

lora_status check_common(lora_dtype dt, int T, int r, int S, int n_slices, const void* meta,
                         size_t meta_bytes) {
  if (dt != LORA_F16 && dt != LORA_BF16) return LORA_ERR_INVALID_ARG;
  if (T < 0 || S < 0 || n_slices < 0) return LORA_ERR_INVALID_ARG;
  if (T > LORA_MAX_TOKENS || S < 1 || S > LORA_MAX_SLOTS) return LORA_ERR_UNSUPPORTED;
  if (n_slices < 1 || n_slices > LORA_MAX_SLICES || !rank_ok(r)) return LORA_ERR_UNSUPPORTED;
  if (meta == nullptr) return LORA_ERR_INVALID_ARG;
  if (!aligned16(meta)) return LORA_ERR_MISALIGNED;
  if (meta_bytes < lora_workspace_bytes(T, S)) return LORA_ERR_INVALID_ARG;
  return LORA_OK;
}

lora_status check_shrink(lora_dtype dt, int T, int D, int r, int S, int n_slices,
                         const void* x, int64_t ldx, const void* const* A, const float* buf,
                         const void* meta, size_t meta_bytes) {
  lora_status s = check_common(dt, T, r, S, n_slices, meta, meta_bytes);
  if (s != LORA_OK) return s;
  if (D <= 0) return LORA_ERR_INVALID_ARG;
  if (T == 0) return LORA_OK;   // nothing to read or write
  if (A == nullptr || x == nullptr || buf == nullptr) return LORA_ERR_INVALID_ARG;
  if (D % 8 != 0) return LORA_ERR_MISALIGNED;
  if (ldx < D) return LORA_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned16(x) || !aligned16(buf)) return LORA_ERR_MISALIGNED;
  for (int i = 0; i < n_slices; ++i) {
    if (A[i] == nullptr) return LORA_ERR_INVALID_ARG;
    if (!aligned16(A[i])) return LORA_ERR_MISALIGNED;
  }
  return LORA_OK;
}

lora_status check_expand(lora_dtype dt, int T, int r, int S, int n_slices, const float* buf,
                         int64_t buf_slice_stride, const void* const* B, const int32_t* D_out,
                         const void* y, int64_t ldy, const int64_t* y_col_off,
                         const void* meta, size_t meta_bytes) {
  lora_status s = check_common(dt, T, r, S, n_slices, meta, meta_bytes);
  if (s != LORA_OK) return s;
  if (T == 0) return LORA_OK;   // nothing to read or write
  if (buf == nullptr || B == nullptr || D_out == nullptr || y == nullptr || y_col_off == nullptr)
    return LORA_ERR_INVALID_ARG;
  if (buf_slice_stride < 0) return LORA_ERR_INVALID_ARG;
  if (buf_slice_stride > 0 && buf_slice_stride < (int64_t)T * r) return LORA_ERR_INVALID_ARG;
  if (buf_slice_stride % 4 != 0 || !aligned16(buf) || !aligned16(y) || ldy % 8 != 0)
    return LORA_ERR_MISALIGNED;
  for (int i = 0; i < n_slices; ++i) {
    if (B[i] == nullptr || D_out[i] <= 0 || y_col_off[i] < 0) return LORA_ERR_INVALID_ARG;
    if (D_out[i] % 8 != 0 || y_col_off[i] % 8 != 0 || !aligned16(B[i]))
      return LORA_ERR_MISALIGNED;
    if (y_col_off[i] + D_out[i] > ldy) return LORA_ERR_INVALID_ARG;
    for (int k = 0; k < i; ++k) {   // output slices must not overlap
      int64_t a0 = y_col_off[i], a1 = a0 + D_out[i];
      int64_t b0 = y_col_off[k], b1 = b0 + D_out[k];
      if (a0 < b1 && b0 < a1) return LORA_ERR_INVALID_ARG;
    }
  }
  return LORA_OK;
}

lora_status check_segments(int T, int n_seg, const int32_t* seg_starts,
                           const int32_t* seg_adapter) {
  if (n_seg < 0 || n_seg > T + 1) return LORA_ERR_INVALID_ARG;
  if (T == 0) return LORA_OK;
  if (seg_starts == nullptr || seg_adapter == nullptr) return LORA_ERR_INVALID_ARG;
  if (n_seg == 0 && T != 0) return LORA_ERR_INVALID_ARG;
  return LORA_OK;
}

int max_items_tokens(int T, int S) { return T / kItemTokens + S + 2; }
int max_items_segments(int T, int n_seg) { return T / kItemTokens + n_seg + 2; }

std::atomic<unsigned long long> g_launches{0};

}  // namespace

namespace lora {
cudaError_t counted_launch(cudaError_t e) {
  if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}
}  // namespace lora

extern "C" {

size_t lora_workspace_bytes(int T, int S) {
  if (T < 0 || T > LORA_MAX_TOKENS || S < 1 || S > LORA_MAX_SLOTS) return 0;
  return MetaLayout(T, S).total;
}

lora_status lora_workspace_reset(void* meta, size_t meta_bytes, lora_stream_t stream) {
  if (meta == nullptr) return LORA_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(meta, 0, meta_bytes, (cudaStream_t)stream));
}

// early: idx is not written by the previous launch on the stream
static lora_status group_impl(int T, int S, const int32_t* idx, void* meta, size_t meta_bytes,
                              lora_stream_t stream, int early) {
  if (T < 0 || S < 0) return LORA_ERR_INVALID_ARG;
  if (T > LORA_MAX_TOKENS || S < 1 || S > LORA_MAX_SLOTS) return LORA_ERR_UNSUPPORTED;
  if (meta == nullptr || (T > 0 && idx == nullptr)) return LORA_ERR_INVALID_ARG;
  if (!aligned16(meta)) return LORA_ERR_MISALIGNED;
  if (meta_bytes < lora_workspace_bytes(T, S)) return LORA_ERR_INVALID_ARG;
  cudaGetLastError();
  return from_cuda(launch_group(T, S, idx, meta, (cudaStream_t)stream, early));
}

lora_status lora_group(int T, int S, const int32_t* idx, void* meta, size_t meta_bytes,
                       lora_stream_t stream) {
  return group_impl(T, S, idx, meta, meta_bytes, stream, 0);
}

lora_status lora_set_slot_ranks(int S, const int32_t* ranks, void* meta, size_t meta_bytes,
                               lora_stream_t stream) {
  if (S < 1 || S > LORA_MAX_SLOTS) return LORA_ERR_UNSUPPORTED;
  if (meta == nullptr) return LORA_ERR_INVALID_ARG;
  if (!aligned16(meta)) return LORA_ERR_MISALIGNED;
  if (meta_bytes < lora_workspace_bytes(0, S)) return LORA_ERR_INVALID_ARG;
  cudaGetLastError();
  return from_cuda(launch_set_ranks(S, ranks, meta, (cudaStream_t)stream));
}

lora_status lora_shrink(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                        const void* x, int64_t ldx, const void* const* A, const int32_t* idx,
                        float* buf, int has_active, const void* meta, size_t meta_bytes,
                        lora_stream_t stream) {
  lora_status s = check_shrink(dtype, T, D, r, S, n_slices, x, ldx, A, buf, meta, meta_bytes);
  if (s != LORA_OK) return s;
  if (!has_active || T == 0) return LORA_OK;
  if (idx == nullptr) return LORA_ERR_INVALID_ARG;
  ShrinkArgs a = {};
  a.x = x;
  a.ldx = ldx;
  for (int i = 0; i < n_slices; ++i) a.A[i] = A[i];
  a.idx = idx;
  a.buf = buf;
  a.T = T; a.D = D; a.r = r; a.S = S; a.n_slices = n_slices;
  a.meta = static_cast<const char*>(meta);
  cudaGetLastError();
  if (grouped_tc_preferred(T, r, S)) {
    cudaError_t e = launch_shrink_grouped_tc(dtype, a, (cudaStream_t)stream);
    if (e != cudaErrorNotSupported) return from_cuda(e);
    cudaGetLastError();
  }
  return from_cuda(launch_shrink_items(dtype, a, max_items_tokens(T, S), (cudaStream_t)stream));
}

lora_status lora_shrink_laned(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                              const void* x, int64_t ldx, const void* const* A,
                              const int32_t* idx, float* buf, int has_active, void* meta,
                              size_t meta_bytes, lora_stream_t stream) {
  // only the workspace's error counters are used
  if (meta == nullptr || meta_bytes < sizeof(MetaHeader)) return LORA_ERR_INVALID_ARG;
  const size_t need = lora_workspace_bytes(T, S);
  lora_status s = check_shrink(dtype, T, D, r, S, n_slices, x, ldx, A, buf, meta,
                               need > meta_bytes ? need : meta_bytes);
  if (s != LORA_OK) return s;
  if (!has_active || T == 0) return LORA_OK;
  if (idx == nullptr) return LORA_ERR_INVALID_ARG;
  ShrinkArgs a = {};
  a.x = x;
  a.ldx = ldx;
  for (int i = 0; i < n_slices; ++i) a.A[i] = A[i];
  a.idx = idx;
  a.buf = buf;
  a.T = T; a.D = D; a.r = r; a.S = S; a.n_slices = n_slices;
  a.meta = static_cast<const char*>(meta);
  cudaGetLastError();
  cudaError_t e = launch_shrink_laned(dtype, a, (cudaStream_t)stream);
  return e == cudaErrorNotSupported ? LORA_ERR_UNSUPPORTED : from_cuda(e);
}

static void fill_expand(ExpandArgs& a, int T, int r, int S, int n_slices, const float* buf,
                        int64_t buf_slice_stride, const void* const* B, const int32_t* D_out,
                        const int32_t* idx, float scale, void* y, int64_t ldy,
                        const int64_t* y_col_off, const void* meta) {
  a.buf = buf;
  a.buf_slice_stride = buf_slice_stride;
  a.idx = idx;
  for (int i = 0; i < n_slices; ++i) {
    a.B[i] = B[i];
    a.D_out[i] = D_out[i];
    a.y_col_off[i] = y_col_off[i];
  }
  a.scale = scale;
  a.y = y;
  a.ldy = ldy;
  a.T = T; a.r = r; a.S = S; a.n_slices = n_slices;
  a.meta = static_cast<const char*>(meta);
}

// after_shrink: the previous launch on the stream is lora_shrink's kernel for
// this batch (lora_bgmv's three-launch path)
static lora_status expand_impl(lora_dtype dtype, int T, int r, int S, int n_slices,
                               const float* buf, int64_t buf_slice_stride, const void* const* B,
                               const int32_t* D_out, const int32_t* idx, float scale, void* y,
                               int64_t ldy, const int64_t* y_col_off, int has_active,
                               const void* meta, size_t meta_bytes, lora_stream_t stream,
                               int after_shrink) {
  lora_status s = check_expand(dtype, T, r, S, n_slices, buf, buf_slice_stride, B, D_out, y,
                               ldy, y_col_off, meta, meta_bytes);
  if (s != LORA_OK) return s;
  if (!has_active || T == 0) return LORA_OK;
  if (idx == nullptr) return LORA_ERR_INVALID_ARG;
  ExpandArgs a = {};
  fill_expand(a, T, r, S, n_slices, buf, buf_slice_stride, B, D_out, idx, scale, y, ldy,
              y_col_off, meta);
  a.after_shrink = after_shrink;
  cudaGetLastError();
  if (grouped_tc_preferred(T, r, S)) {
    cudaError_t e = launch_expand_grouped_tc(dtype, a, (cudaStream_t)stream);
    if (e != cudaErrorNotSupported) return from_cuda(e);
    cudaGetLastError();
  }
  return from_cuda(launch_expand_items(dtype, a, max_items_tokens(T, S), (cudaStream_t)stream));
}

lora_status lora_expand(lora_dtype dtype, int T, int r, int S, int n_slices,
                        const float* buf, int64_t buf_slice_stride, const void* const* B,
                        const int32_t* D_out, const int32_t* idx, float scale, void* y,
                        int64_t ldy, const int64_t* y_col_off, int has_active, const void* meta,
                        size_t meta_bytes, lora_stream_t stream) {
  return expand_impl(dtype, T, r, S, n_slices, buf, buf_slice_stride, B, D_out, idx, scale, y,
                     ldy, y_col_off, has_active, meta, meta_bytes, stream, 0);
}

lora_status lora_shrink_segment(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                                const void* x, int64_t ldx, const void* const* A,
                                const int32_t* seg_starts, const int32_t* seg_adapter,
                                int n_seg, float* buf, int has_active, void* meta,
                                size_t meta_bytes, lora_stream_t stream) {
  lora_status s = check_shrink(dtype, T, D, r, S, n_slices, x, ldx, A, buf, meta, meta_bytes);
  if (s != LORA_OK) return s;
  s = check_segments(T, n_seg, seg_starts, seg_adapter);
  if (s != LORA_OK) return s;
  if (!has_active || T == 0) return LORA_OK;
  ShrinkArgs a = {};
  a.x = x;
  a.ldx = ldx;
  for (int i = 0; i < n_slices; ++i) a.A[i] = A[i];
  a.buf = buf;
  a.T = T; a.D = D; a.r = r; a.S = S; a.n_slices = n_slices;
  a.meta = static_cast<const char*>(meta);
  SegArgs sg = {seg_starts, seg_adapter, n_seg};
  cudaStream_t st = (cudaStream_t)stream;
  cudaGetLastError();
  cudaError_t e = launch_shrink_segment_tc(dtype, a, sg, st);
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    e = launch_segment_items(T, S, n_seg, seg_starts, seg_adapter, meta, st);
    if (e == cudaSuccess) e = launch_shrink_items(dtype, a, max_items_segments(T, n_seg), st);
  }
  return from_cuda(e);
}

// after_shrink: the previous launch on the stream is lora_shrink_segment's
// kernel for this batch (lora_sgmv)
static lora_status expand_segment_impl(lora_dtype dtype, int T, int r, int S, int n_slices,
                                       const float* buf, int64_t buf_slice_stride,
                                       const void* const* B, const int32_t* D_out,
                                       const int32_t* seg_starts, const int32_t* seg_adapter,
                                       int n_seg, float scale, void* y, int64_t ldy,
                                       const int64_t* y_col_off, int has_active, void* meta,
                                       size_t meta_bytes, lora_stream_t stream,
                                       int after_shrink) {
  lora_status s = check_expand(dtype, T, r, S, n_slices, buf, buf_slice_stride, B, D_out, y,
                               ldy, y_col_off, meta, meta_bytes);
  if (s != LORA_OK) return s;
  s = check_segments(T, n_seg, seg_starts, seg_adapter);
  if (s != LORA_OK) return s;
  if (!has_active || T == 0) return LORA_OK;
  ExpandArgs a = {};
  fill_expand(a, T, r, S, n_slices, buf, buf_slice_stride, B, D_out, nullptr, scale, y, ldy,
              y_col_off, meta);
  a.after_shrink = after_shrink;
  SegArgs sg = {seg_starts, seg_adapter, n_seg};
  cudaStream_t st = (cudaStream_t)stream;
  cudaGetLastError();
  cudaError_t e = launch_expand_segment_tc(dtype, a, sg, st);
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    e = launch_segment_items(T, S, n_seg, seg_starts, seg_adapter, meta, st);
    if (e == cudaSuccess) e = launch_expand_items(dtype, a, max_items_segments(T, n_seg), st);
  }
  return from_cuda(e);
}

lora_status lora_expand_segment(lora_dtype dtype, int T, int r, int S, int n_slices,
                                const float* buf, int64_t buf_slice_stride,
                                const void* const* B, const int32_t* D_out,
                                const int32_t* seg_starts, const int32_t* seg_adapter,
                                int n_seg, float scale, void* y, int64_t ldy,
                                const int64_t* y_col_off, int has_active, void* meta,
                                size_t meta_bytes, lora_stream_t stream) {
  return expand_segment_impl(dtype, T, r, S, n_slices, buf, buf_slice_stride, B, D_out,
                             seg_starts, seg_adapter, n_seg, scale, y, ldy, y_col_off, has_active,
                             meta, meta_bytes, stream, 0);
}

lora_status lora_sgmv(lora_dtype dtype, int T, int D, int r, int S, int n_slices, const void* x,
                      int64_t ldx, const void* const* A, int shared_A, const void* const* B,
                      const int32_t* D_out, float scale, void* y, int64_t ldy,
                      const int64_t* y_col_off, float* buf, const int32_t* seg_starts,
                      const int32_t* seg_adapter, int n_seg, int has_active, void* meta,
                      size_t meta_bytes, lora_stream_t stream) {
  const int n_a = shared_A ? 1 : n_slices;
  if (n_slices < 1 || n_slices > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
  if (A == nullptr && T > 0) return LORA_ERR_INVALID_ARG;
  const int64_t stride = shared_A ? 0 : (int64_t)T * r;
  lora_status s = check_shrink(dtype, T, D, r, S, n_a, x, ldx, A, buf, meta, meta_bytes);
  if (s != LORA_OK) return s;
  s = check_expand(dtype, T, r, S, n_slices, buf, stride, B, D_out, y, ldy, y_col_off, meta,
                   meta_bytes);
  if (s != LORA_OK) return s;
  s = check_segments(T, n_seg, seg_starts, seg_adapter);
  if (s != LORA_OK) return s;
  if (!has_active || T == 0) return LORA_OK;
  // the segment shrink launches only kernels that write buf, the workspace's
  // work list and its error counters, none of which the tensor-core expand
  // reads before its wait
  s = lora_shrink_segment(dtype, T, D, r, S, n_a, x, ldx, A, seg_starts, seg_adapter, n_seg, buf,
                          1, meta, meta_bytes, stream);
  if (s != LORA_OK) return s;
  return expand_segment_impl(dtype, T, r, S, n_slices, buf, stride, B, D_out, seg_starts,
                             seg_adapter, n_seg, scale, y, ldy, y_col_off, 1, meta, meta_bytes,
                             stream, 1);
}

static void fill_fused(FusedArgs& f, int T, int D, int r, int S, int n_slices, const void* x,
                       int64_t ldx, const void* const* A, int shared_A, const void* const* B,
                       const int32_t* D_out, float scale, void* y, int64_t ldy,
                       const int64_t* y_col_off, float* buf, const int32_t* idx, void* meta,
                       unsigned flags) {
  f.x = x;
  f.ldx = ldx;
  for (int i = 0; i < n_slices; ++i) {
    f.A[i] = A[shared_A ? 0 : i];
    f.B[i] = B[i];
    f.D_out[i] = D_out[i];
    f.y_col_off[i] = y_col_off[i];
  }
  f.y = y;
  f.ldy = ldy;
  f.buf = buf;
  f.idx = idx;
  MetaHeader* h = static_cast<MetaHeader*>(meta);
  f.bad_index = &h->bad_index;
  f.bad_meta = &h->bad_meta;
  f.T = T; f.D = D; f.r = r; f.S = S; f.n_slices = n_slices;
  f.shared_A = shared_A ? 1 : 0;
  f.scale = scale;
  f.pdl_early = (flags & LORA_FLAG_PDL_EARLY) ? 1 : 0;
}

lora_status lora_bgmv(lora_dtype dtype, int T, int D, int r, int S, int n_slices, const void* x,
                      int64_t ldx, const void* const* A, int shared_A, const void* const* B,
                      const int32_t* D_out, float scale, void* y, int64_t ldy,
                      const int64_t* y_col_off, float* buf, const int32_t* idx, int has_active,
                      unsigned flags, void* meta, size_t meta_bytes, lora_stream_t stream) {
  const int n_a = shared_A ? 1 : n_slices;
  if (n_slices < 1 || n_slices > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
  if (A == nullptr && T > 0) return LORA_ERR_INVALID_ARG;
  lora_status s = check_shrink(dtype, T, D, r, S, n_a, x, ldx, A, buf, meta, meta_bytes);
  if (s != LORA_OK) return s;
  s = check_expand(dtype, T, r, S, n_slices, buf, shared_A ? 0 : (int64_t)T * r, B, D_out, y, ldy,
                   y_col_off, meta, meta_bytes);
  if (s != LORA_OK) return s;
  if (!has_active || T == 0) return LORA_OK;
  if (idx == nullptr) return LORA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  cudaGetLastError();
  FusedArgs f = {};
  fill_fused(f, T, D, r, S, n_slices, x, ldx, A, shared_A, B, D_out, scale, y, ldy, y_col_off,
             buf, idx, meta, flags);
  cudaError_t e = launch_bgmv_fused(dtype, f, st);
  if (e != cudaErrorNotSupported) return from_cuda(e);
  cudaGetLastError();
  if (!(flags & LORA_FLAG_GROUPED)) {
    s = group_impl(T, S, idx, meta, meta_bytes, stream, (flags & LORA_FLAG_PDL_EARLY) ? 1 : 0);
    if (s != LORA_OK) return s;
  }
  // a successful lora_shrink is exactly one launch on `stream`: the expand's
  // predecessor
  s = lora_shrink(dtype, T, D, r, S, n_a, x, ldx, A, idx, buf, 1, meta, meta_bytes, stream);
  if (s != LORA_OK) return s;
  return expand_impl(dtype, T, r, S, n_slices, buf, shared_A ? 0 : (int64_t)T * r, B, D_out,
                     idx, scale, y, ldy, y_col_off, 1, meta, meta_bytes, stream, 1);
}

int lora_bgmv_launches(lora_dtype dtype, int T, int D, int r, int S, int n_slices,
                       const int32_t* D_out) {
  if (dtype != LORA_F16 && dtype != LORA_BF16) return LORA_ERR_INVALID_ARG;
  if (T < 0 || D <= 0 || n_slices < 1 || n_slices > LORA_MAX_SLICES || !rank_ok(r) || S < 1 ||
      S > LORA_MAX_SLOTS || D_out == nullptr)
    return LORA_ERR_UNSUPPORTED;
  return bgmv_fused_fits(T, D, r, n_slices, D_out) ? 1 : 3;
}

lora_status lora_check_errors(void* meta, size_t meta_bytes, lora_stream_t stream) {
  if (meta == nullptr || meta_bytes < sizeof(MetaHeader)) return LORA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LORA_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpy(h, meta, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return LORA_ERR_CUDA;
  if (h[0] || h[1]) {
    int z[2] = {0, 0};
    if (cudaMemcpy(meta, z, sizeof(z), cudaMemcpyHostToDevice) != cudaSuccess)
      return LORA_ERR_CUDA;
    return LORA_ERR_BAD_INDEX;
  }
  return LORA_OK;
}

const char* lora_status_string(lora_status status) {
  switch (status) {
    case LORA_OK: return "LORA_OK";
    case LORA_ERR_INVALID_ARG: return "LORA_ERR_INVALID_ARG";
    case LORA_ERR_UNSUPPORTED: return "LORA_ERR_UNSUPPORTED";
    case LORA_ERR_MISALIGNED: return "LORA_ERR_MISALIGNED";
    case LORA_ERR_CUDA: return "LORA_ERR_CUDA";
    case LORA_ERR_BAD_INDEX: return "LORA_ERR_BAD_INDEX";
  }
  return "LORA_ERR_UNKNOWN";
}

const char* lora_build_info(void) { return "liblora_b200 sm_100a 0.2"; }

unsigned long long lora_launch_count(void) {
  return g_launches.load(std::memory_order_relaxed);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free per-token shrink.
//
// For callers that cannot allocate device memory themselves: code running
// where cudaMalloc is unavailable or forbidden (inside a CUDA-graph capture
// that must not allocate, an allocator hook, a plugin host that hands out
// only input and output buffers) and so cannot provide the workspace that
// lora_group / lora_shrink need.  This entry point keeps that workspace in a
// fixed device array instead.
// ---------------------------------------------------------------------------
namespace {

// Sized for LORA_NOALLOC_MAX_TOKENS tokens over LORA_MAX_SLOTS slots; every
// GPU that loads the library holds it until the process exits.
constexpr size_t kNoallocScratchBytes = 246784;
static_assert(kNoallocScratchBytes == LORA_NOALLOC_SCRATCH_BYTES, "header and library agree");
static __device__ __align__(256) char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_noalloc_ptr[kMaxDevices];

// Device address of the scratch array for the current device.  The array's
// name in host code is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" LORA_API lora_status lora_shrink_noalloc(lora_dtype dtype, int T, int D, int r, int S,
                                                    int n_slices, const void* x, int64_t ldx,
                                                    const void* const* A, const int32_t* idx,
                                                    float* buf, int has_active,
                                                    lora_stream_t stream) {
  if (T > LORA_NOALLOC_MAX_TOKENS) return LORA_ERR_UNSUPPORTED;
  if (T >= 0 && S >= 1 && S <= LORA_MAX_SLOTS &&
      MetaLayout(T, S).total > kNoallocScratchBytes)
    return LORA_ERR_UNSUPPORTED;
  // validate against a stand-in workspace size first: nothing is touched yet
  static const char kFakeMeta[16] __attribute__((aligned(16))) = {0};
  lora_status s = check_shrink(dtype, T, D, r, S, n_slices, x, ldx, A, buf, kFakeMeta,
                               kNoallocScratchBytes);
  if (s != LORA_OK) return s;
  if (!has_active || T == 0) return LORA_OK;
  if (idx == nullptr) return LORA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  cudaGetLastError();
  if (noalloc_scratch(&scratch) != cudaSuccess) return LORA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  // the header (error counters, item count) must start at zero each call
  cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(MetaHeader), st);
  if (e == cudaSuccess) e = launch_group(T, S, idx, scratch, st);
  if (e != cudaSuccess) return LORA_ERR_CUDA;
  ShrinkArgs a = {};
  a.x = x;
  a.ldx = ldx;
  for (int i = 0; i < n_slices; ++i) a.A[i] = A[i];
  a.idx = idx;
  a.buf = buf;
  a.T = T; a.D = D; a.r = r; a.S = S; a.n_slices = n_slices;
  a.meta = static_cast<const char*>(scratch);
  return from_cuda(launch_shrink_items(dtype, a, max_items_tokens(T, S), st));
}
