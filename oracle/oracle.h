/*
 * oracle.h -- plain, slow CPU executor of op streams.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. The GPU runtime never calls it and
 * shares no code with it.
 *
 * What it computes: each op of a stream, one after another in submission order
 * (one valid topological order of the dependency DAG), written as the plain
 * definition of the op in double precision and rounded once to the output
 * type. The persistent kernel of GPUOS (arXiv 2604.17861, abstract) claims to
 * run the same ops as one-launch-per-op execution, only without the launches,
 * so the definition of each op is the whole specification.
 *
 * Memory model: all fp32 tensors live in one float arena, all bf16 tensors in
 * one uint16 arena (bf16 bit patterns). Ops name operands by element offsets.
 */
#ifndef ORACLE_H
#define ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  ORC_F32 = 0,
  ORC_BF16 = 1
};

enum {
  ORC_K_ADD = 101,
  ORC_K_MUL,
  ORC_K_SCALE,
  ORC_K_GELU,
  ORC_K_RELU_AFFINE,
  ORC_K_SILU_MUL,
  ORC_K_EW_CHAIN,
  ORC_K_ROWSUM,
  ORC_K_ROWMAX,
  ORC_K_SOFTMAX,
  ORC_K_RMSNORM,
  ORC_K_LAYERNORM,
  ORC_K_ROTARY
};

/* micro-ops of a fused elementwise chain; accumulator starts as operand 0 */
enum {
  ORC_M_AFFINE = 1, /* acc = fmaf(s[k], acc, s[k+1]), k += 2 */
  ORC_M_SCALE,      /* acc = acc * s[k], k += 1 */
  ORC_M_ADDS,       /* acc = acc + s[k], k += 1 */
  ORC_M_RELU,
  ORC_M_GELU,
  ORC_M_SILU,
  ORC_M_ADD1,
  ORC_M_MUL1,
  ORC_M_ADD2,
  ORC_M_MUL2
};

typedef struct {
  int32_t kind;      /* ORC_K_* */
  int32_t dtype;     /* ORC_F32 / ORC_BF16, for all operands and the output */
  int64_t in_off[3]; /* element offsets into the arena of dtype; -1 = unused */
  int64_t out_off;
  int64_t rows, cols;
  int64_t in_n[2];   /* element counts of operands 0 and 1 (modulo broadcast) */
  float s[4];        /* scalars, meaning per kind */
  int32_t pos;       /* rotary position */
  int32_t nprog;     /* chain length */
  int8_t prog[8];    /* ORC_M_* */
} orc_op;

/* Status codes */
enum { ORC_OK = 0, ORC_EBOUNDS = -1, ORC_EKIND = -2, ORC_EPROG = -3 };

/* Runs ops[0..nops) in order; reads and writes the arenas in place.
 * Returns ORC_OK, or the negated index-1 of the first bad op combined with a
 * status in *bad_op / return value. */
int orc_run(const orc_op* ops, int64_t nops, float* a32, int64_t n32,
            uint16_t* a16, int64_t n16, int64_t* bad_op);

/* Applies one op to operands read from the arenas, writing its whole output to
 * `out` (float* or uint16_t* by dtype) instead of the arena. Used to check a
 * GPU op on the GPU's own inputs. */
int orc_apply(const orc_op* op, const float* a32, int64_t n32,
              const uint16_t* a16, int64_t n16, void* out);

/* Element helpers, exposed for the pins. */
uint16_t orc_f32_to_bf16(float f);
float orc_bf16_to_f32(uint16_t h);
double orc_gelu(double x);

#ifdef __cplusplus
}
#endif
#endif
