/*
 * oracle.c -- plain CPU executor of op streams (test infrastructure only).
 *
 * Every op is its textbook definition evaluated in double precision and
 * rounded once to the output type, except where an op is defined by fp32
 * steps (the affine micro-op is a single-rounding fmaf; a fused chain rounds
 * its accumulator to fp32 after every micro-op, as a register-resident chain
 * does). Ops run in submission order.
 *
 * Sources of each definition:
 *  - relu(a*x+b): "Launch Overhead and Fusion", section "Fusion" (the fused
 *    multiply, add, relu chain) and the worked example of that page's demo.
 *  - add, mul, scale, gelu (erf form), silu*mul, row sum/max, softmax,
 *    RMSNorm, LayerNorm, rotary (half-split pairs, base 10000): the pages name
 *    only the classes of ops (the GPUOS page, "The Paper": many small tensor
 *    ops of inference and attention); the formulas are the standard
 *    definitions.
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared oracle.c -lm
 */
#include "oracle.h"

#include <math.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) /* NaN: keep sign and payload top, force quiet */
    return (uint16_t)((u >> 16) | 0x0040u);
  /* round to nearest, ties to even: add half an ulp minus one, plus the lsb */
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

float orc_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ---------------------------------------------------------------- scalar defs */
double orc_gelu(double x) {
  /* 0.5 x (1 + erf(x/sqrt2)) written with erfc so the negative tail keeps
   * its relative accuracy */
  return 0.5 * x * erfc(-x / sqrt(2.0));
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static float relu_f(float v) { return (v <= 0.0f) ? 0.0f : v; } /* NaN passes, -0 -> +0 */

/* ---------------------------------------------------------------- arena access */
typedef struct {
  int dtype;
  float* a32;
  const float* c32;
  int64_t n32;
  uint16_t* a16;
  const uint16_t* c16;
  int64_t n16;
} arenas;

static double ld(const arenas* A, int64_t off) {
  if (A->dtype == ORC_F32) return (double)A->c32[off];
  return (double)orc_bf16_to_f32(A->c16[off]);
}

static float ldf(const arenas* A, int64_t off) {
  if (A->dtype == ORC_F32) return A->c32[off];
  return orc_bf16_to_f32(A->c16[off]);
}

/* rounds a double once to the op's output type and stores it */
static void st(int dtype, void* out, int64_t idx, double v) {
  float f = (float)v;
  if (dtype == ORC_F32)
    ((float*)out)[idx] = f;
  else
    ((uint16_t*)out)[idx] = orc_f32_to_bf16(f);
}

static int in_bounds(const arenas* A, int64_t off, int64_t n) {
  int64_t cap = (A->dtype == ORC_F32) ? A->n32 : A->n16;
  return off >= 0 && n >= 0 && off + n <= cap;
}

/* ---------------------------------------------------------------- ops */
static int check_op(const orc_op* op, const arenas* A, int want_out_arena) {
  int64_t n = op->rows * op->cols;
  if (op->rows < 1 || op->cols < 1) return ORC_EBOUNDS;
  int64_t out_n = (op->kind == ORC_K_ROWSUM || op->kind == ORC_K_ROWMAX) ? op->rows : n;
  if (want_out_arena && !in_bounds(A, op->out_off, out_n)) return ORC_EBOUNDS;
  switch (op->kind) {
    case ORC_K_ADD:
    case ORC_K_MUL:
    case ORC_K_SILU_MUL:
      if (op->in_n[0] < 1 || op->in_n[1] < 1) return ORC_EBOUNDS;
      if (!in_bounds(A, op->in_off[0], op->in_n[0]) || !in_bounds(A, op->in_off[1], op->in_n[1]))
        return ORC_EBOUNDS;
      return ORC_OK;
    case ORC_K_SCALE:
    case ORC_K_GELU:
    case ORC_K_RELU_AFFINE:
      if (op->in_n[0] < 1 || !in_bounds(A, op->in_off[0], op->in_n[0])) return ORC_EBOUNDS;
      return ORC_OK;
    case ORC_K_EW_CHAIN: {
      if (op->nprog < 0 || op->nprog > 8) return ORC_EPROG;
      if (op->in_n[0] < 1 || !in_bounds(A, op->in_off[0], op->in_n[0])) return ORC_EBOUNDS;
      int nsc = 0;
      for (int p = 0; p < op->nprog; ++p) {
        int m = op->prog[p];
        if (m == ORC_M_AFFINE) nsc += 2;
        else if (m == ORC_M_SCALE || m == ORC_M_ADDS) nsc += 1;
        else if (m == ORC_M_ADD1 || m == ORC_M_MUL1) {
          if (op->in_n[1] < 1 || !in_bounds(A, op->in_off[1], op->in_n[1])) return ORC_EBOUNDS;
        } else if (m == ORC_M_ADD2 || m == ORC_M_MUL2) {
          if (!in_bounds(A, op->in_off[2], n)) return ORC_EBOUNDS;
        } else if (m < ORC_M_AFFINE || m > ORC_M_MUL2)
          return ORC_EPROG;
      }
      if (nsc > 4) return ORC_EPROG;
      return ORC_OK;
    }
    case ORC_K_ROWSUM:
    case ORC_K_ROWMAX:
    case ORC_K_SOFTMAX:
      return in_bounds(A, op->in_off[0], n) ? ORC_OK : ORC_EBOUNDS;
    case ORC_K_RMSNORM:
      return (in_bounds(A, op->in_off[0], n) && in_bounds(A, op->in_off[1], op->cols)) ? ORC_OK
                                                                                         : ORC_EBOUNDS;
    case ORC_K_LAYERNORM:
      return (in_bounds(A, op->in_off[0], n) && in_bounds(A, op->in_off[1], op->cols) &&
              in_bounds(A, op->in_off[2], op->cols))
                 ? ORC_OK
                 : ORC_EBOUNDS;
    case ORC_K_ROTARY:
      if (op->cols % 2) return ORC_EBOUNDS;
      return in_bounds(A, op->in_off[0], n) ? ORC_OK : ORC_EBOUNDS;
    default:
      return ORC_EKIND;
  }
}

/* One fused-chain element: fp32 accumulator rounded after every micro-op. */
static float chain_elem(const orc_op* op, const arenas* A, int64_t e) {
  int64_t n = op->rows * op->cols;
  float acc = ldf(A, op->in_off[0] + e % op->in_n[0]);
  int k = 0;
  for (int p = 0; p < op->nprog; ++p) {
    switch (op->prog[p]) {
      case ORC_M_AFFINE:
        acc = fmaf(op->s[k], acc, op->s[k + 1]);
        k += 2;
        break;
      case ORC_M_SCALE:
        acc = (float)((double)acc * (double)op->s[k]);
        k += 1;
        break;
      case ORC_M_ADDS:
        acc = (float)((double)acc + (double)op->s[k]);
        k += 1;
        break;
      case ORC_M_RELU:
        acc = relu_f(acc);
        break;
      case ORC_M_GELU:
        acc = (float)orc_gelu((double)acc);
        break;
      case ORC_M_SILU:
        acc = (float)((double)acc * sigmoid((double)acc));
        break;
      case ORC_M_ADD1:
        acc = (float)((double)acc + ld(A, op->in_off[1] + e % op->in_n[1]));
        break;
      case ORC_M_MUL1:
        acc = (float)((double)acc * ld(A, op->in_off[1] + e % op->in_n[1]));
        break;
      case ORC_M_ADD2:
        acc = (float)((double)acc + ld(A, op->in_off[2] + e % n));
        break;
      case ORC_M_MUL2:
        acc = (float)((double)acc * ld(A, op->in_off[2] + e % n));
        break;
    }
  }
  return acc;
}

/* Computes op, writing the output through `out` (arena or scratch). The
 * input arenas must not alias `out` for row ops unless out == the op's own
 * output slot in the arena (row ops read a whole row before writing it). */
static void exec_op(const orc_op* op, const arenas* A, void* out, int64_t out_base) {
  const int64_t rows = op->rows, cols = op->cols, n = rows * cols;
  const int dt = op->dtype;
  switch (op->kind) {
    case ORC_K_ADD:
      for (int64_t e = 0; e < n; ++e)
        st(dt, out, out_base + e,
           ld(A, op->in_off[0] + e % op->in_n[0]) + ld(A, op->in_off[1] + e % op->in_n[1]));
      break;
    case ORC_K_MUL:
      for (int64_t e = 0; e < n; ++e)
        st(dt, out, out_base + e,
           ld(A, op->in_off[0] + e % op->in_n[0]) * ld(A, op->in_off[1] + e % op->in_n[1]));
      break;
    case ORC_K_SCALE:
      for (int64_t e = 0; e < n; ++e)
        st(dt, out, out_base + e, (double)op->s[0] * ld(A, op->in_off[0] + e % op->in_n[0]));
      break;
    case ORC_K_GELU:
      for (int64_t e = 0; e < n; ++e)
        st(dt, out, out_base + e, orc_gelu(ld(A, op->in_off[0] + e % op->in_n[0])));
      break;
    case ORC_K_RELU_AFFINE:
      for (int64_t e = 0; e < n; ++e) {
        float v = fmaf(op->s[0], ldf(A, op->in_off[0] + e % op->in_n[0]), op->s[1]);
        st(dt, out, out_base + e, (double)relu_f(v));
      }
      break;
    case ORC_K_SILU_MUL:
      for (int64_t e = 0; e < n; ++e) {
        double g = ld(A, op->in_off[0] + e % op->in_n[0]);
        double u = ld(A, op->in_off[1] + e % op->in_n[1]);
        st(dt, out, out_base + e, g * sigmoid(g) * u);
      }
      break;
    case ORC_K_EW_CHAIN:
      for (int64_t e = 0; e < n; ++e) st(dt, out, out_base + e, (double)chain_elem(op, A, e));
      break;
    case ORC_K_ROWSUM:
      for (int64_t r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < cols; ++c) acc += ld(A, op->in_off[0] + r * cols + c);
        st(dt, out, out_base + r, acc);
      }
      break;
    case ORC_K_ROWMAX:
      for (int64_t r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int64_t c = 0; c < cols; ++c) {
          double v = ld(A, op->in_off[0] + r * cols + c);
          if (v > m) m = v; /* NaN elements are skipped */
        }
        st(dt, out, out_base + r, m);
      }
      break;
    case ORC_K_SOFTMAX:
      for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = op->in_off[0] + r * cols;
        double m = -INFINITY, sum = 0.0;
        for (int64_t c = 0; c < cols; ++c) {
          double v = ld(A, base + c);
          if (v > m) m = v;
        }
        for (int64_t c = 0; c < cols; ++c) sum += exp(ld(A, base + c) - m);
        /* read all values of the row before writing (in-place safe) */
        double tmp[8192];
        int64_t c0 = 0;
        while (c0 < cols) {
          int64_t c1 = c0 + 8192 < cols ? c0 + 8192 : cols;
          for (int64_t c = c0; c < c1; ++c) tmp[c - c0] = exp(ld(A, base + c) - m) / sum;
          for (int64_t c = c0; c < c1; ++c) st(dt, out, out_base + r * cols + c, tmp[c - c0]);
          c0 = c1;
        }
      }
      break;
    case ORC_K_RMSNORM:
      for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = op->in_off[0] + r * cols;
        double ss = 0.0;
        for (int64_t c = 0; c < cols; ++c) {
          double v = ld(A, base + c);
          ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)cols + (double)op->s[0]);
        for (int64_t c = 0; c < cols; ++c)
          st(dt, out, out_base + r * cols + c, ld(A, base + c) * inv * ld(A, op->in_off[1] + c));
      }
      break;
    case ORC_K_LAYERNORM:
      for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = op->in_off[0] + r * cols;
        double mu = 0.0, var = 0.0;
        for (int64_t c = 0; c < cols; ++c) mu += ld(A, base + c);
        mu /= (double)cols;
        for (int64_t c = 0; c < cols; ++c) {
          double d = ld(A, base + c) - mu;
          var += d * d;
        }
        var /= (double)cols; /* biased */
        double inv = 1.0 / sqrt(var + (double)op->s[0]);
        for (int64_t c = 0; c < cols; ++c)
          st(dt, out, out_base + r * cols + c,
             (ld(A, base + c) - mu) * inv * ld(A, op->in_off[1] + c) + ld(A, op->in_off[2] + c));
      }
      break;
    case ORC_K_ROTARY: {
      const int64_t half = cols / 2;
      for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = op->in_off[0] + r * cols;
        for (int64_t i = 0; i < half; ++i) {
          double theta = pow((double)op->s[0], -2.0 * (double)i / (double)cols);
          double phi = (double)op->pos * theta;
          double c = cos(phi), s = sin(phi);
          double x1 = ld(A, base + i), x2 = ld(A, base + i + half);
          st(dt, out, out_base + r * cols + i, x1 * c - x2 * s);
          st(dt, out, out_base + r * cols + i + half, x2 * c + x1 * s);
        }
      }
      break;
    }
  }
}

int orc_run(const orc_op* ops, int64_t nops, float* a32, int64_t n32, uint16_t* a16, int64_t n16,
            int64_t* bad_op) {
  for (int64_t i = 0; i < nops; ++i) {
    arenas A = {ops[i].dtype, a32, a32, n32, a16, a16, n16};
    int rc = check_op(&ops[i], &A, 1);
    if (rc != ORC_OK) {
      if (bad_op) *bad_op = i;
      return rc;
    }
    void* out = (ops[i].dtype == ORC_F32) ? (void*)a32 : (void*)a16;
    exec_op(&ops[i], &A, out, ops[i].out_off);
  }
  return ORC_OK;
}

int orc_apply(const orc_op* op, const float* a32, int64_t n32, const uint16_t* a16, int64_t n16,
              void* out) {
  arenas A = {op->dtype, 0, a32, n32, 0, a16, n16};
  int rc = check_op(op, &A, 0);
  if (rc != ORC_OK) return rc;
  exec_op(op, &A, out, 0);
  return ORC_OK;
}
