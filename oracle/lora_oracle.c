/*
 * Oracle for the multi-LoRA shrink / expand path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or table with the CUDA
 * library in gather_matmul_b200/csrc.
 *
 * What it computes is the plain definition, in double precision, one token
 * at a time, with no blocking, fusion or reordering:
 *
 *   shrink   buf[i][t][j] = sum_d x[t][d] * A_i[idx[t]][j][d]
 *   expand   y[t][off_i + o] = y_old[t][off_i + o]
 *                              + scale * sum_j buf[i][t][j] * B_i[idx[t]][o][j]
 *
 * Source: "[Hardware][TPU][V1] Better tpu multilora compilation"
 * (vllm-project/vllm pull 16989), the ref_bgmv baseline posted in the
 * discussion: the adapter matrices are gathered per token by its index
 * (selected = loras[idxs]) and each token's input vector is multiplied by its
 * own selected [L, D] matrix, giving a [T, L] result.  Shrink is that
 * operation with loras = A; expand is the same operation with loras = B
 * applied to the shrink result, scaled and added into the output slice.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - index -1 means "base model only" ("Add multi-LoRA support", vllm pull
 *    1804, Features list: LoRA and non-LoRA requests share one batch).  Such
 *    a token gets buf = 0 and its y row is left as it was.  ref_bgmv's
 *    loras[-1] would wrap to the last slot; that Python negative indexing is
 *    deliberately NOT reproduced.
 *  - an index outside [-1, S) is treated like -1 and counted as bad.
 *  - the intermediate is kept unrounded here (fp64); the pull-1804
 *    Limitations list names a half-precision intermediate as an accuracy loss.
 *  - one scale per call multiplies the expand sum.
 *  - segments: seg_starts is CSR [n_seg + 1], starting at 0 and ending at T,
 *    non-decreasing; token t in [seg_starts[s], seg_starts[s+1]) uses adapter
 *    seg_adapter[s].  The segment form is the same computation with idx
 *    expanded from the segments.
 *
 * Element decoding of fp16 / bf16 is written from the IEEE 754 binary16
 * definition and from bfloat16's definition (the upper half of a binary32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { LO_F16 = 0, LO_BF16 = 1 };

static int lo_threads = 1;

/* Number of host threads the per-token loops may use (tokens are
 * independent, so this never changes a result). */
int lo_set_threads(int n) {
#ifdef _OPENMP
  lo_threads = n > 0 ? n : 1;
  return lo_threads;
#else
  (void)n;
  lo_threads = 1;
  return 1;
#endif
}

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double dec_f16(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)f, -24);                 /* 0.f * 2^(1-15) */
  } else if (e == 31) {
    v = f ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + f), e - 25);     /* 1.f * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
static double dec_bf16(uint16_t b) {
  int sign = (b >> 15) & 1;
  int e = (b >> 7) & 0xff;
  int f = b & 0x7f;
  double v;
  if (e == 0) {
    v = ldexp((double)f, -133);                /* 0.f * 2^(1-127) */
  } else if (e == 255) {
    v = f ? NAN : INFINITY;
  } else {
    v = ldexp((double)(128 + f), e - 134);     /* 1.f * 2^(e-127) */
  }
  return sign ? -v : v;
}

/* Every 16-bit pattern decoded once with the definitions above, then looked
 * up (the values are the same; the table only avoids re-deriving them for
 * each of the billions of products at full size). */
static double table_f16[65536], table_bf16[65536];
static int tables_ready = 0;

static void init_tables(void) {
  if (tables_ready) return;
  for (int b = 0; b < 65536; ++b) {
    table_f16[b] = dec_f16((uint16_t)b);
    table_bf16[b] = dec_bf16((uint16_t)b);
  }
  tables_ready = 1;
}

static double dec(int dtype, uint16_t bits) {
  return dtype == LO_BF16 ? table_bf16[bits] : table_f16[bits];
}

double lo_decode(int dtype, uint16_t bits) {
  return dtype == LO_BF16 ? dec_bf16(bits) : dec_f16(bits);
}

void lo_decode_array(int dtype, const uint16_t* in, double* out, int64_t n) {
  init_tables();
  for (int64_t k = 0; k < n; ++k) out[k] = dec(dtype, in[k]);
}

/* Adapter of token t, with anything outside [0, S) mapped to "no adapter". */
static int adapter_of(const int32_t* idx, int t, int S) {
  int a = idx[t];
  return (a >= 0 && a < S) ? a : -1;
}

static int count_bad(int T, int S, const int32_t* idx) {
  int bad = 0;
  for (int t = 0; t < T; ++t)
    if (idx[t] < -1 || idx[t] >= S) ++bad;
  return bad;
}

/*
 * Group-by-slot metadata: a stable counting sort of the active tokens by
 * adapter slot.  slot_off[S+1] is the exclusive prefix of per-slot counts,
 * perm[slot_off[g] .. slot_off[g+1]) lists the tokens of slot g in
 * increasing token order, n_active = slot_off[S].  Returns the number of bad
 * indices (those are left out, like -1).
 */
int lo_group_by_slot(int T, int S, const int32_t* idx, int32_t* perm,
                     int32_t* slot_off, int32_t* n_active) {
  for (int g = 0; g <= S; ++g) slot_off[g] = 0;
  for (int t = 0; t < T; ++t) {
    int a = adapter_of(idx, t, S);
    if (a >= 0) slot_off[a + 1] += 1;
  }
  for (int g = 0; g < S; ++g) slot_off[g + 1] += slot_off[g];
  int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)(S > 0 ? S : 1));
  for (int g = 0; g < S; ++g) fill[g] = slot_off[g];
  for (int t = 0; t < T; ++t) {
    int a = adapter_of(idx, t, S);
    if (a >= 0) perm[fill[a]++] = t;
  }
  free(fill);
  *n_active = slot_off[S];
  return count_bad(T, S, idx);
}

/*
 * Shrink, one slice at a time, one token at a time:
 *   buf[i][t][j] = sum over d of x[t][d] * A_i[idx[t]][j][d]     (fp64)
 * cabs (optional) receives sum over d of |x[t][d] * A_i[idx[t]][j][d]|, the
 * magnitude a floating-point error bound scales with.
 * x is [T, ldx] row-major, A_i is [S, r, D] contiguous.  Tokens without an
 * adapter get buf = 0.  Returns the number of bad indices.
 */
int lo_shrink(int dtype, int T, int D, int r, int S, int n_slices,
              const uint16_t* x, int64_t ldx, const uint16_t* const* A,
              const int32_t* idx, double* buf, double* cabs) {
  init_tables();
  for (int i = 0; i < n_slices; ++i) {
    const uint16_t* Ai = A[i];
#pragma omp parallel for num_threads(lo_threads) schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
      double* out = buf + ((int64_t)i * T + t) * r;
      double* mag = cabs ? cabs + ((int64_t)i * T + t) * r : NULL;
      int a = adapter_of(idx, t, S);
      for (int j = 0; j < r; ++j) {
        double s = 0.0, m = 0.0;
        if (a >= 0) {
          const uint16_t* row = Ai + ((int64_t)a * r + j) * D;   /* selected[j][:] */
          const uint16_t* xt = x + (int64_t)t * ldx;
          for (int d = 0; d < D; ++d) {
            double p = dec(dtype, xt[d]) * dec(dtype, row[d]);
            s += p;
            m += fabs(p);
          }
        }
        out[j] = s;
        if (mag) mag[j] = m;
      }
    }
  }
  return count_bad(T, S, idx);
}

/*
 * Expand into fused output slices:
 *   y[t][off_i + o] = y_old[t][off_i + o]
 *                     + scale * sum over j of buf_i[t][j] * B_i[idx[t]][o][j]
 * buf_i starts at buf + i * buf_slice_stride (stride 0: all slices share one
 * [T, r] intermediate) and is [T, r].  B_i is [S, D_out[i], r] contiguous.
 * y_old is [T, ldy] fp16/bf16 bits; y_out is [T, ldy] fp64, a copy of y_old
 * with the sums added.  Rows of tokens without an adapter, and columns no
 * slice covers, are y_old unchanged.  Returns the number of bad indices.
 */
int lo_expand(int dtype, int T, int r, int S, int n_slices, const double* buf,
              int64_t buf_slice_stride, const uint16_t* const* B,
              const int32_t* D_out, const int32_t* idx, double scale,
              const uint16_t* y_old, int64_t ldy, const int64_t* y_col_off,
              double* y_out) {
  init_tables();
#pragma omp parallel for num_threads(lo_threads) schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    for (int64_t c = 0; c < ldy; ++c)
      y_out[(int64_t)t * ldy + c] = dec(dtype, y_old[(int64_t)t * ldy + c]);
    int a = adapter_of(idx, t, S);
    if (a < 0) continue;
    for (int i = 0; i < n_slices; ++i) {
      const double* bt = buf + (int64_t)i * buf_slice_stride + (int64_t)t * r;
      const uint16_t* Bi = B[i];
      for (int o = 0; o < D_out[i]; ++o) {
        const uint16_t* row = Bi + ((int64_t)a * D_out[i] + o) * r;  /* selected[o][:] */
        double s = 0.0;
        for (int j = 0; j < r; ++j) s += bt[j] * dec(dtype, row[j]);
        y_out[(int64_t)t * ldy + y_col_off[i] + o] += scale * s;
      }
    }
  }
  return count_bad(T, S, idx);
}

/*
 * Segment metadata to per-token indices.  Returns 0 on success, -1 if the
 * segments are malformed (seg_starts[0] != 0, decreasing, or last != T).
 */
int lo_segments_to_idx(int T, int n_seg, const int32_t* seg_starts,
                       const int32_t* seg_adapter, int32_t* idx) {
  if (n_seg < 0) return -1;
  if (seg_starts[0] != 0 || seg_starts[n_seg] != T) return -1;
  for (int s = 0; s < n_seg; ++s)
    if (seg_starts[s + 1] < seg_starts[s]) return -1;
  for (int s = 0; s < n_seg; ++s)
    for (int t = seg_starts[s]; t < seg_starts[s + 1]; ++t) idx[t] = seg_adapter[s];
  return 0;
}

/* Segment forms: the same computation on idx expanded from the segments.
 * Returns -1000 for malformed segments, else the number of bad adapters'
 * tokens. */
int lo_shrink_segment(int dtype, int T, int D, int r, int S, int n_slices,
                      const uint16_t* x, int64_t ldx, const uint16_t* const* A,
                      const int32_t* seg_starts, const int32_t* seg_adapter,
                      int n_seg, double* buf, double* cabs) {
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
  int rc = lo_segments_to_idx(T, n_seg, seg_starts, seg_adapter, idx);
  if (rc == 0) rc = lo_shrink(dtype, T, D, r, S, n_slices, x, ldx, A, idx, buf, cabs);
  else rc = -1000;
  free(idx);
  return rc;
}

int lo_expand_segment(int dtype, int T, int r, int S, int n_slices,
                      const double* buf, int64_t buf_slice_stride,
                      const uint16_t* const* B, const int32_t* D_out,
                      const int32_t* seg_starts, const int32_t* seg_adapter,
                      int n_seg, double scale, const uint16_t* y_old,
                      int64_t ldy, const int64_t* y_col_off, double* y_out) {
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
  int rc = lo_segments_to_idx(T, n_seg, seg_starts, seg_adapter, idx);
  if (rc == 0)
    rc = lo_expand(dtype, T, r, S, n_slices, buf, buf_slice_stride, B, D_out, idx,
                   scale, y_old, ldy, y_col_off, y_out);
  else rc = -1000;
  free(idx);
  return rc;
}
