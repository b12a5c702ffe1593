// ops.cuh -- op bodies: one work item of one op, run by a group of warps.
//
// The same bodies serve the persistent kernel (its compute warps) and the
// one-kernel-per-op baseline, so both paths compute identical results. A body
// sees the op's ring entry in shared memory, the item index, and a compute
// context (thread index within the group, group size, a named barrier and a
// small shared scratch). Elementwise items stream 16-byte vectors with several
// loads in flight per thread; row items give each warp a row segment, reduce
// with warp shuffles and combine segments through shared memory.
#pragma once

#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace gpuos_impl {

// Shared-memory staging area of one compute warp: three stages, each armed
// through its own mbarrier and filled by bulk asynchronous copies (the TMA
// engine, no tensor map, no multicast).
constexpr int WS_STAGES = 3;
constexpr int WS_STAGE_BYTES = 4096;
constexpr int WS_BYTES = WS_STAGES * WS_STAGE_BYTES;
struct __align__(128) WarpSmem {
  unsigned char buf[WS_BYTES];
  unsigned long long bar[WS_STAGES];
  unsigned seq;  // stage uses so far, modulo 6: use u lives in stage u % 3 with phase parity (u / 3) & 1
};

// Rotation angles of the last rotary op this CTA ran: cos and sin of
// pos * base^(-2i/cols) for each column pair i. Consecutive rotary ops with the
// same base, width and position (q and k of every layer of a decode step) reuse
// them instead of recomputing them in double precision.
constexpr int ROT_MAX_PAIRS = 256;
struct RotCache {
  float base;
  int pos;
  long long cols;  // 0: empty
  double2 cs[ROT_MAX_PAIRS];
};

struct Cx {
  int tid, nthr;       // thread index in the compute group, group size
  int warp, nwarps, lane;
  int bar;             // named barrier id of the compute group
  float4* part;        // shared scratch, >= nwarps entries
  WarpSmem* ws;        // this warp's staging area
  DevState* st;        // error reporting (null in the one-kernel-per-op baseline)
  HostCtl* hctl;
  u64 id;              // op id, for error reports
  u32 flags;           // KF_* of the launch (KF_NO_BULK: register paths only)
  RotCache* rot;       // shared rotary angle cache, or null
};

struct OpEnv {
  DevState* st;        // null in the one-kernel-per-op baseline
  HostCtl* hctl;
  u64 timeout_ns;
  u64 id;
};

__device__ __forceinline__ void cx_sync(const Cx& c) { bar_sync(c.bar, c.nthr); }

// First device error wins; it is mirrored to the host control block, then the
// abort flag tells every CTA to leave.
static __device__ __noinline__ void raise_error(DevState* st, HostCtl* hctl, unsigned code, u64 id) {
  if (st == nullptr) return;
  u64 word = (u64)code | ((id + 1) << 8);
  u64 old = atomicCAS(&st->err.v, 0ull, word);
  if (old == 0) {
    hctl->err_id = id;
    fence_acq_rel_sys();
    st_relaxed_sys32(&hctl->status, code);
  }
  st_release_gpu(&st->abort_.v, 1ull);
}

// ------------------------------------------------------------------ elements
__device__ __forceinline__ float bf2f(unsigned short h) { return __uint_as_float((unsigned)h << 16); }
__device__ __forceinline__ unsigned short f2bf(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }
__device__ __forceinline__ bool al16(u64 p) { return (p & 15ull) == 0; }

// 8 consecutive elements starting at element i (i % 8 == 0, base 16-byte aligned)
template <int DT>
__device__ __forceinline__ void ld8(u64 base, long long i, float (&v)[8]) {
  if (DT == 0) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i);
    float4 a = __ldcg(p), b = __ldcg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    uint4 r = __ldcg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned short*>(base) + i));
    unsigned w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
}
template <int DT>
__device__ __forceinline__ void st8(u64 base, long long i, const float (&v)[8]) {
  if (DT == 0) {
    float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + i);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 r;
    r.x = (unsigned)f2bf(v[0]) | ((unsigned)f2bf(v[1]) << 16);
    r.y = (unsigned)f2bf(v[2]) | ((unsigned)f2bf(v[3]) << 16);
    r.z = (unsigned)f2bf(v[4]) | ((unsigned)f2bf(v[5]) << 16);
    r.w = (unsigned)f2bf(v[6]) | ((unsigned)f2bf(v[7]) << 16);
    *reinterpret_cast<uint4*>(reinterpret_cast<unsigned short*>(base) + i) = r;
  }
}
template <int DT>
__device__ __forceinline__ float ld1(u64 base, long long i) {
  if (DT == 0) return __ldcg(reinterpret_cast<const float*>(base) + i);
  return bf2f(__ldcg(reinterpret_cast<const unsigned short*>(base) + i));
}
template <int DT>
__device__ __forceinline__ void st1(u64 base, long long i, float v) {
  if (DT == 0)
    reinterpret_cast<float*>(base)[i] = v;
  else
    reinterpret_cast<unsigned short*>(base)[i] = f2bf(v);
}

// ------------------------------------------------------------------ staged (shared-memory) access
__device__ __forceinline__ void lds8_f32(unsigned a, float (&v)[8]) {
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]) : "r"(a));
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]) : "r"(a + 16));
}
// 8 elements at shared byte address a
template <int DT>
__device__ __forceinline__ void lds8(unsigned a, float (&v)[8]) {
  if (DT == 0) {
    lds8_f32(a, v);
  } else {
    unsigned w0, w1, w2, w3;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3) : "r"(a));
    const unsigned w[4] = {w0, w1, w2, w3};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
}
template <int DT>
__device__ __forceinline__ float lds1(unsigned a) {
  if (DT == 0) {
    float f;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f) : "r"(a));
    return f;
  }
  unsigned short h;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(a));
  return bf2f(h);
}

// Waits for stage use u of this warp's staging area, bounded by one second;
// a copy that never lands is reported (GPUOS_ETIMEDOUT) instead of hanging.
static __device__ __noinline__ void ws_wait_fail(const Cx cx) {
  if (cx.lane == 0) raise_error(cx.st, cx.hctl, GPUOS_ETIMEDOUT, cx.id);
}
__device__ __forceinline__ void ws_wait(const Cx& cx, unsigned u) {
  unsigned long long* b = &cx.ws->bar[u % WS_STAGES];
  const unsigned par = (u / WS_STAGES) & 1u;
  if (mbar_try_wait(b, par)) return;
  const u64 t0 = globaltimer();
  for (unsigned spins = 0;; ++spins) {
    if (mbar_try_wait(b, par)) return;
    if ((spins & 1023) == 1023) {
      if (cx.st && ld_relaxed_gpu(&cx.st->abort_.v)) return;  // another CTA failed: stop waiting
      if (globaltimer() - t0 > 1000000000ull) {
        ws_wait_fail(cx);
        return;
      }
    }
  }
}
__device__ __forceinline__ unsigned ws_addr(const Cx& cx, unsigned byte_off) { return smem_u32(cx.ws->buf) + byte_off; }

// ------------------------------------------------------------------ scalar defs
__device__ __forceinline__ float relu_f(float v) { return (v <= 0.0f) ? 0.0f : v; }  // NaN passes, -0 -> +0
// The double-precision transcendentals stay out of line: inlined into the
// unrolled vector loops they would multiply register pressure for every op.
static __device__ __noinline__ float gelu_f(float x) {
  double xd = (double)x;
  return (float)(0.5 * xd * erfc(-xd / 1.4142135623730951));
}
// gelu of the standalone fp32 op: 0.5 x erfc(t) at t = -x/sqrt(2), with t
// carried as a float plus its rounding error dt (the exact product error by
// fma, and the low part of 1/sqrt(2)), and erfc corrected to first order,
// erfc(t + dt) = erfc(t) - (2/sqrt(pi)) exp(-t^2) dt. Without dt the relative
// error of erfc would grow like 2 t^2 2^-24 (1e-6 at |x| = 4.2); with it the
// error is that of erfcf (4 ulp by CUDA's documentation) plus two roundings,
// under 1e-6 relative. For x >= 6, Phi(x) > 1 - 2^-26 and x Phi(x) rounds
// to x; for |x| < 1e-30, Phi(x) = 1/2 far below an ulp; x < -10 (where the
// result nears the subnormal range), -inf and NaN take the double path.
__device__ __forceinline__ float gelu_fast(float x) {
  if (x >= 6.0f) return x;
  if (fabsf(x) < 1e-30f) return 0.5f * x;
  if (!(x >= -10.0f)) return gelu_f(x);
  const float c_hi = 0.70710677f, c_lo = 1.2101617e-08f;  // 1/sqrt(2) = c_hi + c_lo
  const float nx = -x;
  const float t = __fmul_rn(nx, c_hi);
  const float dt = __fadd_rn(__fmaf_rn(nx, c_hi, -t), __fmul_rn(nx, c_lo));
  const float r = erfcf(t) - 1.1283791671f * __expf(-t * t) * dt;
  return 0.5f * x * r;
}
static __device__ __noinline__ float silu_f(float x) {
  double xd = (double)x;
  return (float)(xd / (1.0 + exp(-xd)));
}
static __device__ __noinline__ float silu_mul_f(float g, float u) {
  double gd = (double)g;
  return (float)(gd / (1.0 + exp(-gd)) * (double)u);
}

// exp for softmax: the hardware 2^t approximation (ex2.approx.f32: relative
// error about 2^-22, subnormal results kept) at t = x log2(e). Rounding t costs
// a relative error of |t| 2^-24 ln 2 in the result, about 1e-6 at the
// x >= -25 that softmax rows of moderate spread reach: far inside the 1e-4 bound.
__device__ __forceinline__ float sm_exp(float x) {
  float r;
  asm("ex2.approx.f32 %0, %1;" : "=f"(r) : "f"(x * 1.4426950408889634f));
  return r;
}

// silu(g) * u for bf16 outputs, whose bound (2 bf16 ulp) leaves room for fp32
// with the hardware exp; large |g| keeps the double path.
__device__ __forceinline__ float silu_mul_bf(float g, float u) {
  if (fabsf(g) > 80.0f) return silu_mul_f(g, u);
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// Fused micro-op program over one element; the program and scalars are read
// from the shared-memory entry (uniform across the group).
__device__ __forceinline__ float chain_f(const RingEntry& E, float acc, float x1, float x2) {
  int k = 0;
  const int nm = E.nmicro;
  for (int i = 0; i < nm; ++i) {
    switch (E.micro[i]) {
      case GPUOS_M_AFFINE: acc = __fmaf_rn(E.s[k & 3], acc, E.s[(k + 1) & 3]); k += 2; break;
      case GPUOS_M_SCALE: acc = __fmul_rn(acc, E.s[k & 3]); k += 1; break;
      case GPUOS_M_ADDS: acc = __fadd_rn(acc, E.s[k & 3]); k += 1; break;
      case GPUOS_M_RELU: acc = relu_f(acc); break;
      case GPUOS_M_GELU: acc = gelu_f(acc); break;
      case GPUOS_M_SILU: acc = silu_f(acc); break;
      case GPUOS_M_ADD1: acc = __fadd_rn(acc, x1); break;
      case GPUOS_M_MUL1: acc = __fmul_rn(acc, x1); break;
      case GPUOS_M_ADD2: acc = __fadd_rn(acc, x2); break;
      case GPUOS_M_MUL2: acc = __fmul_rn(acc, x2); break;
      default: break;
    }
  }
  return acc;
}

template <int OPK, int DT = 0>
__device__ __forceinline__ float ew_f(const RingEntry& E, float x0, float x1, float x2) {
  if (OPK == GPUOS_OP_ADD) return __fadd_rn(x0, x1);
  if (OPK == GPUOS_OP_MUL) return __fmul_rn(x0, x1);
  if (OPK == GPUOS_OP_SCALE) return __fmul_rn(E.s[0], x0);
  if (OPK == GPUOS_OP_GELU) return gelu_fast(x0);
  if (OPK == GPUOS_OP_RELU_AFFINE) return relu_f(__fmaf_rn(E.s[0], x0, E.s[1]));
  if (OPK == GPUOS_OP_SILU_MUL) return DT == 1 ? silu_mul_bf(x0, x1) : silu_mul_f(x0, x1);
  return chain_f(E, x0, x1, x2);  // GPUOS_OP_EW_CHAIN, OPK_CHAIN_CALLS
}

// Program-wide micro-op loop for one vector of 8 elements: the micro-op
// switch is taken once per vector instead of once per element.
__device__ __forceinline__ void chain8(const RingEntry& E, float (&a)[8], const float (&x1)[8],
                                       const float (&x2)[8]) {
  int k = 0;
  const int nm = E.nmicro;
  for (int i = 0; i < nm; ++i) {
    const int m = E.micro[i];
    if (m == GPUOS_M_AFFINE) {
      const float s0 = E.s[k & 3], s1 = E.s[(k + 1) & 3];
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fmaf_rn(s0, a[j], s1);
      k += 2;
    } else if (m == GPUOS_M_RELU) {
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = relu_f(a[j]);
    } else if (m == GPUOS_M_SCALE) {
      const float s0 = E.s[k & 3];
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fmul_rn(a[j], s0);
      k += 1;
    } else if (m == GPUOS_M_ADDS) {
      const float s0 = E.s[k & 3];
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fadd_rn(a[j], s0);
      k += 1;
    } else if (m == GPUOS_M_ADD1) {
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fadd_rn(a[j], x1[j]);
    } else if (m == GPUOS_M_MUL1) {
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fmul_rn(a[j], x1[j]);
    } else if (m == GPUOS_M_ADD2) {
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fadd_rn(a[j], x2[j]);
    } else if (m == GPUOS_M_MUL2) {
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fmul_rn(a[j], x2[j]);
    }
  }
}

__device__ __forceinline__ void chain_uses(const RingEntry& E, bool& u1, bool& u2) {
  u1 = u2 = false;
  for (int i = 0; i < E.nmicro; ++i) {
    const int m = E.micro[i];
    u1 |= (m == GPUOS_M_ADD1 || m == GPUOS_M_MUL1);
    u2 |= (m == GPUOS_M_ADD2 || m == GPUOS_M_MUL2);
  }
}

constexpr int EW_UNR = 2;  // tiles in flight per warp (binary ops; unary ops use twice as many)

// Pseudo-opcode: a fused program that calls an out-of-line transcendental
// (gelu, silu) runs element by element, without the unrolled vector batch.
constexpr int OPK_CHAIN_CALLS = 1000;

// e mod m, in 32 bits when both fit
__device__ __forceinline__ u64 umod(u64 a, u64 m) {
  if (((a | m) >> 32) == 0) return (u64)((u32)a % (u32)m);
  return a % m;
}

// Register-path tiles: a warp takes 256 consecutive elements at a time.
// Vector layout (all operands direct and 16-byte aligned): lane l holds
// fp32 elements 4l..4l+3 and 128+4l..128+4l+3 (two float4, each warp load
// one contiguous 512 bytes), or bf16 elements 8l..8l+7 (one 16-byte load).
// Scalar layout (a broadcast or unaligned operand): lane l holds elements
// l, l+32, ..., l+224, each warp load one contiguous 128 (64) bytes.
constexpr int EW_TILE = 256;

template <int DT>
__device__ __forceinline__ void tile_ld(u64 base, long long t0, int lane, float (&v)[8]) {
  if (DT == 0) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + t0);
    const float4 a = __ldcg(p + lane), b = __ldcg(p + 32 + lane);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    ld8<1>(base, t0 + 8 * lane, v);
  }
}
template <int DT>
__device__ __forceinline__ void tile_st(u64 base, long long t0, int lane, const float (&v)[8]) {
  if (DT == 0) {
    float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + t0);
    p[lane] = make_float4(v[0], v[1], v[2], v[3]);
    p[32 + lane] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    st8<1>(base, t0 + 8 * lane, v);
  }
}

// Scalar layout of one operand of m elements read at index e mod m (m == n:
// direct). j starts at (t0 + lane) mod m and steps by step = 32 mod m.
template <int DT>
__device__ __forceinline__ void tile_gather(u64 base, long long t0, int lane, long long m, long long n,
                                            long long step, long long e1, float (&v)[8]) {
  long long j = (m == n) ? t0 + lane : (long long)umod((u64)(t0 + lane), (u64)m);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[k] = (t0 + lane + 32 * k < e1) ? ld1<DT>(base, j) : 0.f;
    j += step;
    if (j >= m) j -= m;
  }
}

template <int DT, int OPK>
__device__ __forceinline__ void ew_apply8(const RingEntry& E, float (&a)[8], const float (&b)[8],
                                          const float (&c)[8]) {
  if (OPK == GPUOS_OP_EW_CHAIN) {
    chain8(E, a, b, c);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) a[j] = ew_f<OPK, DT>(E, a[j], b[j], c[j]);
  }
}

// Each body is out of line: inlined together into one dispatcher, the union
// of their unrolled register arrays would spill.
// CH: which extra operands the body reads (bit 0: in1, bit 1: in2), or -1 to
// decide at run time from the fused program. UNR: tiles in flight per warp.
template <int DT, int OPK, int UNR, int CH>
static __device__ __noinline__ void ew_loop(const RingEntry& E, u32 item, u32 elem_chunk, const Cx cx) {
  const long long n = E.rows * E.cols;
  const long long e0 = (long long)item * elem_chunk;
  const long long e1 = min(n, e0 + (long long)elem_chunk);
  bool u1, u2;
  if (CH < 0) {
    chain_uses(E, u1, u2);
  } else {
    u1 = (CH & 1) != 0;
    u2 = (CH & 2) != 0;
  }
  const long long n0 = E.in_n0, n1 = E.in_n1;
  const bool vec = n0 == n && al16(E.in0) && (!u1 || (n1 == n && al16(E.in1))) && (!u2 || al16(E.in2)) &&
                   al16(E.out);
  const int lane = cx.lane, w = cx.warp, NW = cx.nwarps;
  const long long full = (e1 - e0) / EW_TILE, tiles = (e1 - e0 + EW_TILE - 1) / EW_TILE;
  long long t = w;
  if (vec) {
    for (; t + (long long)(UNR - 1) * NW < full; t += (long long)UNR * NW) {
      float a[UNR][8], b[UNR][8], c[UNR][8];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const long long t0 = e0 + (t + (long long)u * NW) * EW_TILE;
        tile_ld<DT>(E.in0, t0, lane, a[u]);
#pragma unroll
        for (int j = 0; j < 8; ++j) b[u][j] = c[u][j] = 0.f;
        if (u1) tile_ld<DT>(E.in1, t0, lane, b[u]);
        if (u2) tile_ld<DT>(E.in2, t0, lane, c[u]);
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        ew_apply8<DT, OPK>(E, a[u], b[u], c[u]);
        tile_st<DT>(E.out, e0 + (t + (long long)u * NW) * EW_TILE, lane, a[u]);
      }
    }
    for (; t < full; t += NW) {
      const long long t0 = e0 + t * EW_TILE;
      float a[8], b[8], c[8];
      tile_ld<DT>(E.in0, t0, lane, a);
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = c[j] = 0.f;
      if (u1) tile_ld<DT>(E.in1, t0, lane, b);
      if (u2) tile_ld<DT>(E.in2, t0, lane, c);
      ew_apply8<DT, OPK>(E, a, b, c);
      tile_st<DT>(E.out, t0, lane, a);
    }
    // t is now the first tile >= full that this warp owns: the partial last
    // tile, if any, takes the scalar layout below
  }
  const long long s0 = n0 < n ? (long long)umod(32, (u64)n0) : 32;
  const long long s1 = (u1 && n1 < n) ? (long long)umod(32, (u64)n1) : 32;
  for (; t < tiles; t += NW) {
    const long long t0 = e0 + t * EW_TILE;
    float a[8], b[8], c[8];
    tile_gather<DT>(E.in0, t0, lane, n0, n, s0, e1, a);
#pragma unroll
    for (int j = 0; j < 8; ++j) b[j] = c[j] = 0.f;
    if (u1) tile_gather<DT>(E.in1, t0, lane, n1, n, s1, e1, b);
    if (u2) tile_gather<DT>(E.in2, t0, lane, n, n, 32, e1, c);
    ew_apply8<DT, OPK>(E, a, b, c);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const long long e = t0 + lane + 32 * k;
      if (e < e1) st1<DT>(E.out, e, a[k]);
    }
  }
}

// Elementwise item through this warp's staging area: the item is cut into
// chunks of 2 KB per operand; warp w takes chunks w, w + nwarps, ...; lane 0
// keeps three chunks in flight with bulk copies while the warp computes the
// oldest from shared memory and stores straight to global memory. Operands
// 0 and (if CH) 1 are staged; they must be direct (no broadcast) and 16-byte
// aligned, as must the output. The op's ragged end (< 16 bytes) is read from
// global memory.
constexpr int EW_CHUNK_BYTES = WS_STAGE_BYTES / 2;

template <int DT, int OPK, int CH>
static __device__ __noinline__ void ew_stream(const RingEntry& E, u32 item, u32 elem_chunk, const Cx cx) {
  constexpr int ES = DT == 0 ? 4 : 2;
  constexpr int CE = EW_CHUNK_BYTES / ES;  // elements per chunk
  const long long n = E.rows * E.cols;
  const long long e0 = (long long)item * elem_chunk;
  const long long e1 = min(n, e0 + (long long)elem_chunk);
  const long long nchunks = (e1 - e0 + CE - 1) / CE;
  const int w = cx.warp, NW = cx.nwarps, lane = cx.lane;
  const int mine = nchunks > w ? (int)((u32)(nchunks - w + NW - 1) / (u32)NW) : 0;  // nchunks <= elem_chunk / 256
  if (mine == 0) return;
  const unsigned base = cx.ws->seq;
  __syncwarp();
  auto issue = [&](int t) {  // lane 0 only
    const long long e = e0 + (long long)(w + t * NW) * CE;
    const long long ne = min((long long)CE, e1 - e);
    const unsigned bytes = (unsigned)((ne * ES) & ~15ll);
    const unsigned u = base + (unsigned)t;
    unsigned long long* b = &cx.ws->bar[u % WS_STAGES];
    unsigned char* dst = cx.ws->buf + (u % WS_STAGES) * WS_STAGE_BYTES;
    mbar_arrive_expect_tx(b, CH ? 2 * bytes : bytes);
    if (bytes) {
      bulk_g2s(dst, reinterpret_cast<const unsigned char*>(E.in0) + e * ES, bytes, b);
      if (CH) bulk_g2s(dst + EW_CHUNK_BYTES, reinterpret_cast<const unsigned char*>(E.in1) + e * ES, bytes, b);
    }
  };
  if (lane == 0) {
    fence_proxy_async_global();  // outputs of earlier ops were written through the generic proxy
    for (int t = 0; t < mine && t < WS_STAGES; ++t) issue(t);
  }
  for (int t = 0; t < mine; ++t) {
    const unsigned u = base + (unsigned)t;
    const long long e = e0 + (long long)(w + t * NW) * CE;
    const long long ne = min((long long)CE, e1 - e);
    const long long staged = ((ne * ES) & ~15ll) / ES;  // elements that arrived by bulk copy
    ws_wait(cx, u);
    const unsigned a0 = ws_addr(cx, (u % WS_STAGES) * WS_STAGE_BYTES);
#pragma unroll
    for (int k = 0; k < CE / 8 / 32; ++k) {
      const int blk = lane + 32 * k;
      const long long eb = blk * 8;  // element offset within the chunk
      if (eb >= ne) continue;
      float x[8], y[8], z[8];
      if (eb + 8 <= staged) {
        lds8<DT>(a0 + (unsigned)(eb * ES), x);
        if (CH) lds8<DT>(a0 + EW_CHUNK_BYTES + (unsigned)(eb * ES), y);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const long long ej = eb + j;
          x[j] = ej < staged ? lds1<DT>(a0 + (unsigned)(ej * ES)) : (ej < ne ? ld1<DT>(E.in0, e + ej) : 0.f);
          if (CH) y[j] = ej < staged ? lds1<DT>(a0 + EW_CHUNK_BYTES + (unsigned)(ej * ES)) : (ej < ne ? ld1<DT>(E.in1, e + ej) : 0.f);
        }
      }
      if (!CH) {
#pragma unroll
        for (int j = 0; j < 8; ++j) y[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) z[j] = 0.f;
      if (OPK == GPUOS_OP_EW_CHAIN) {
        chain8(E, x, y, z);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = ew_f<OPK, DT>(E, x[j], y[j], 0.f);
      }
      if (eb + 8 <= ne) {
        st8<DT>(E.out, e + eb, x);
      } else {
        for (int j = 0; j < 8 && eb + j < ne; ++j) st1<DT>(E.out, e + eb + j, x[j]);
      }
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
    if (lane == 0 && t + WS_STAGES < mine) issue(t + WS_STAGES);
  }
  if (lane == 0) cx.ws->seq = (base + (unsigned)mine) % (2 * WS_STAGES);
  __syncwarp();
}

// A fused pair (see M_STORE1): scalar micro-ops only, with one store of the
// intermediate accumulator to in1. Both outputs are written, as two separate
// ops would write them.
__device__ __forceinline__ bool chain_has_store(const RingEntry& E) {
  bool st = false;
  for (int i = 0; i < E.nmicro; ++i) st |= E.micro[i] == M_STORE1;
  return st;
}
__device__ __forceinline__ void chain8_store(const RingEntry& E, float (&a)[8], float (&mid)[8]) {
  int k = 0;
  const int nm = E.nmicro;
  for (int i = 0; i < nm; ++i) {
    const int m = E.micro[i];
    if (m == GPUOS_M_AFFINE) {
      const float s0 = E.s[k & 3], s1 = E.s[(k + 1) & 3];
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fmaf_rn(s0, a[j], s1);
      k += 2;
    } else if (m == GPUOS_M_RELU) {
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = relu_f(a[j]);
    } else if (m == GPUOS_M_SCALE) {
      const float s0 = E.s[k & 3];
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fmul_rn(a[j], s0);
      k += 1;
    } else if (m == GPUOS_M_ADDS) {
      const float s0 = E.s[k & 3];
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = __fadd_rn(a[j], s0);
      k += 1;
    } else if (m == M_STORE1) {
#pragma unroll
      for (int j = 0; j < 8; ++j) mid[j] = a[j];
    }
  }
}

// Body of a fused pair: one item of whole or ragged tiles, in0 read once,
// the intermediate written to in1 and the result to out.
template <int DT>
static __device__ __noinline__ void ew_fused(const RingEntry& E, u32 item, u32 elem_chunk, const Cx cx) {
  const long long n = E.rows * E.cols;
  const long long e0 = (long long)item * elem_chunk;
  const long long e1 = min(n, e0 + (long long)elem_chunk);
  const long long n0 = E.in_n0;
  const bool vec = n0 == n && al16(E.in0) && al16(E.in1) && al16(E.out);
  const int lane = cx.lane, w = cx.warp, NW = cx.nwarps;
  const long long full = (e1 - e0) / EW_TILE, tiles = (e1 - e0 + EW_TILE - 1) / EW_TILE;
  long long t = w;
  if (vec) {
    for (; t + NW < full; t += 2ll * NW) {
      float a[2][8], mid[2][8];
#pragma unroll
      for (int u = 0; u < 2; ++u) tile_ld<DT>(E.in0, e0 + (t + (long long)u * NW) * EW_TILE, lane, a[u]);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const long long t0 = e0 + (t + (long long)u * NW) * EW_TILE;
        chain8_store(E, a[u], mid[u]);
        tile_st<DT>(E.in1, t0, lane, mid[u]);
        tile_st<DT>(E.out, t0, lane, a[u]);
      }
    }
    for (; t < full; t += NW) {
      const long long t0 = e0 + t * EW_TILE;
      float a[8], mid[8];
      tile_ld<DT>(E.in0, t0, lane, a);
      chain8_store(E, a, mid);
      tile_st<DT>(E.in1, t0, lane, mid);
      tile_st<DT>(E.out, t0, lane, a);
    }
  }
  const long long s0 = n0 < n ? (long long)umod(32, (u64)n0) : 32;
  for (; t < tiles; t += NW) {
    const long long t0 = e0 + t * EW_TILE;
    float a[8], mid[8];
    tile_gather<DT>(E.in0, t0, lane, n0, n, s0, e1, a);
    chain8_store(E, a, mid);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const long long e = t0 + lane + 32 * k;
      if (e < e1) {
        st1<DT>(E.in1, e, mid[k]);
        st1<DT>(E.out, e, a[k]);
      }
    }
  }
}

__device__ __forceinline__ bool chain_calls(const RingEntry& E) {
  bool c = false;
  for (int i = 0; i < E.nmicro; ++i) c |= (E.micro[i] == GPUOS_M_GELU || E.micro[i] == GPUOS_M_SILU);
  return c;
}

template <int DT>
__device__ void ew_item(const RingEntry& E, u32 item, u32 elem_chunk, const Cx& cx) {
  const long long n = E.rows * E.cols;
  if (E.opcode == GPUOS_OP_EW_CHAIN && chain_has_store(E)) {
    ew_fused<DT>(E, item, elem_chunk, cx);
    return;
  }
  // Bulk-copy staging pays off when the whole grid streams one large op from
  // HBM (an op of several items); a single-item op is latency-bound on one SM,
  // where the register path's loads arrive sooner.
  const bool s0 = E.in_n0 == n && al16(E.in0) && !(cx.flags & KF_NO_BULK) && n > (long long)elem_chunk;
  const bool s1 = E.in_n1 == n && al16(E.in1);
  if (s0 && al16(E.out)) {
    bool u1 = false, u2 = false;
    if (E.opcode == GPUOS_OP_EW_CHAIN) chain_uses(E, u1, u2);
    const bool bin = E.opcode == GPUOS_OP_ADD || E.opcode == GPUOS_OP_MUL || E.opcode == GPUOS_OP_SILU_MUL;
    if (!u2 && (!(bin || u1) || s1)) {
      switch (E.opcode) {
        case GPUOS_OP_ADD: ew_stream<DT, GPUOS_OP_ADD, 1>(E, item, elem_chunk, cx); return;
        case GPUOS_OP_MUL: ew_stream<DT, GPUOS_OP_MUL, 1>(E, item, elem_chunk, cx); return;
        case GPUOS_OP_SCALE: ew_stream<DT, GPUOS_OP_SCALE, 0>(E, item, elem_chunk, cx); return;
        case GPUOS_OP_GELU: ew_stream<DT, GPUOS_OP_GELU, 0>(E, item, elem_chunk, cx); return;
        case GPUOS_OP_RELU_AFFINE: ew_stream<DT, GPUOS_OP_RELU_AFFINE, 0>(E, item, elem_chunk, cx); return;
        case GPUOS_OP_SILU_MUL: ew_stream<DT, GPUOS_OP_SILU_MUL, 1>(E, item, elem_chunk, cx); return;
        default:
          if (chain_calls(E)) break;  // fused programs with out-of-line calls keep the register path
          if (u1)
            ew_stream<DT, GPUOS_OP_EW_CHAIN, 1>(E, item, elem_chunk, cx);
          else
            ew_stream<DT, GPUOS_OP_EW_CHAIN, 0>(E, item, elem_chunk, cx);
          return;
      }
    }
  }
  switch (E.opcode) {
    case GPUOS_OP_ADD: ew_loop<DT, GPUOS_OP_ADD, EW_UNR, 1>(E, item, elem_chunk, cx); break;
    case GPUOS_OP_MUL: ew_loop<DT, GPUOS_OP_MUL, EW_UNR, 1>(E, item, elem_chunk, cx); break;
    case GPUOS_OP_SCALE: ew_loop<DT, GPUOS_OP_SCALE, 2 * EW_UNR, 0>(E, item, elem_chunk, cx); break;
    case GPUOS_OP_GELU: ew_loop<DT, GPUOS_OP_GELU, 1, 0>(E, item, elem_chunk, cx); break;
    case GPUOS_OP_RELU_AFFINE: ew_loop<DT, GPUOS_OP_RELU_AFFINE, 2 * EW_UNR, 0>(E, item, elem_chunk, cx); break;
    case GPUOS_OP_SILU_MUL: ew_loop<DT, GPUOS_OP_SILU_MUL, EW_UNR, 1>(E, item, elem_chunk, cx); break;
    default:
      if (chain_calls(E)) {
        ew_loop<DT, OPK_CHAIN_CALLS, 1, -1>(E, item, elem_chunk, cx);
      } else {
        bool u1, u2;
        chain_uses(E, u1, u2);
        const int ch = (u1 ? 1 : 0) | (u2 ? 2 : 0);
        if (ch == 0)
          ew_loop<DT, GPUOS_OP_EW_CHAIN, 2 * EW_UNR, 0>(E, item, elem_chunk, cx);
        else if (ch == 1)
          ew_loop<DT, GPUOS_OP_EW_CHAIN, EW_UNR, 1>(E, item, elem_chunk, cx);
        else if (ch == 2)
          ew_loop<DT, GPUOS_OP_EW_CHAIN, EW_UNR, 2>(E, item, elem_chunk, cx);
        else
          ew_loop<DT, GPUOS_OP_EW_CHAIN, EW_UNR / 2, 3>(E, item, elem_chunk, cx);
      }
      break;
  }
}

// ------------------------------------------------------------------ row ops
struct Acc {
  float a, b;
};

__device__ __forceinline__ Acc acc_init(int op) {
  if (op == GPUOS_OP_ROWMAX || op == GPUOS_OP_SOFTMAX) return Acc{-INFINITY, 0.f};
  return Acc{0.f, 0.f};
}

// Folds 8 elements into a partial row statistic.
__device__ __forceinline__ void acc8(int op, Acc& A, const float (&x)[8], float K) {
  if (op == GPUOS_OP_ROWSUM) {
#pragma unroll
    for (int j = 0; j < 8; ++j) A.a += x[j];
  } else if (op == GPUOS_OP_ROWMAX) {
#pragma unroll
    for (int j = 0; j < 8; ++j) A.a = fmaxf(A.a, x[j]);
  } else if (op == GPUOS_OP_SOFTMAX) {
    float m = A.a;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, x[j]);
    float s = (A.a == -INFINITY) ? 0.f : A.b * sm_exp(A.a - m);
#pragma unroll
    for (int j = 0; j < 8; ++j) s += sm_exp(x[j] - m);
    A.a = m;
    A.b = s;
  } else if (op == GPUOS_OP_RMSNORM) {
#pragma unroll
    for (int j = 0; j < 8; ++j) A.a = __fmaf_rn(x[j], x[j], A.a);
  } else {  // LAYERNORM: shifted sums
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float d = x[j] - K;
      A.a += d;
      A.b = __fmaf_rn(d, d, A.b);
    }
  }
}
__device__ __forceinline__ void acc1(int op, Acc& A, float x, float K) {
  if (op == GPUOS_OP_ROWSUM) {
    A.a += x;
  } else if (op == GPUOS_OP_ROWMAX) {
    A.a = fmaxf(A.a, x);
  } else if (op == GPUOS_OP_SOFTMAX) {
    const float m = fmaxf(A.a, x);
    A.b = ((A.a == -INFINITY) ? 0.f : A.b * sm_exp(A.a - m)) + sm_exp(x - m);
    A.a = m;
  } else if (op == GPUOS_OP_RMSNORM) {
    A.a = __fmaf_rn(x, x, A.a);
  } else {
    const float d = x - K;
    A.a += d;
    A.b = __fmaf_rn(d, d, A.b);
  }
}
__device__ __forceinline__ void acc_merge(int op, Acc& A, const Acc& B) {
  if (op == GPUOS_OP_ROWMAX) {
    A.a = fmaxf(A.a, B.a);
  } else if (op == GPUOS_OP_SOFTMAX) {
    const float m = fmaxf(A.a, B.a);
    if (m != -INFINITY) {
      A.b = A.b * sm_exp(A.a - m) + B.b * sm_exp(B.a - m);
      A.a = m;
    }
  } else {
    A.a += B.a;
    A.b += B.b;
  }
}
__device__ __forceinline__ void acc_warp(int op, Acc& A) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    Acc B{__shfl_xor_sync(0xffffffffu, A.a, off), __shfl_xor_sync(0xffffffffu, A.b, off)};
    acc_merge(op, A, B);
  }
}

// Writes the outputs of columns [c0, c1) of one row from its full statistic.
// Per-row constants of the output pass from the row's full statistic:
// softmax (max, sum), RMSNorm (1/rms, -), LayerNorm (mean, 1/std).
__device__ __forceinline__ void row_consts(int op, const Acc& A, float K, long long cols, float eps, float& p0,
                                           float& p1) {
  p0 = 0.f;
  p1 = 0.f;
  if (op == GPUOS_OP_SOFTMAX) {
    p0 = A.a;
    p1 = 1.0f / A.b;  // one division per row; outputs multiply
  } else if (op == GPUOS_OP_RMSNORM) {
    p0 = 1.0f / sqrtf(A.a / (float)cols + eps);
  } else if (op == GPUOS_OP_LAYERNORM) {
    const float mean_d = A.a / (float)cols;
    float var = (A.b - A.a * mean_d) / (float)cols;
    var = fmaxf(var, 0.f);
    p0 = K + mean_d;
    p1 = 1.0f / sqrtf(var + eps);
  }
}

__device__ __forceinline__ void row_apply8(int op, float p0, float p1, const float (&x)[8], const float (&w)[8],
                                           const float (&b)[8], float (&y)[8]) {
  if (op == GPUOS_OP_SOFTMAX) {
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(sm_exp(x[j] - p0), p1);
  } else if (op == GPUOS_OP_RMSNORM) {
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(__fmul_rn(x[j], p0), w[j]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = __fmaf_rn(__fmul_rn(x[j] - p0, p1), w[j], b[j]);
  }
}

// Folds columns [lo, hi) of a row (element rb + lo 16-byte aligned, hi - lo
// a multiple of 8) into A: whole 256-column tiles in the tile layout, U at a
// time, the rest as 8 consecutive columns per lane.
template <int DT, int U>
__device__ __forceinline__ void acc_span(int op, Acc& A, float K, u64 base, long long rb, long long lo, long long hi,
                                         int lane) {
  long long c = lo;
  for (; c + (long long)U * EW_TILE <= hi; c += (long long)U * EW_TILE) {
    float x[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) tile_ld<DT>(base, rb + c + u * EW_TILE, lane, x[u]);
#pragma unroll
    for (int u = 0; u < U; ++u) acc8(op, A, x[u], K);
  }
  for (; c + EW_TILE <= hi; c += EW_TILE) {
    float x[8];
    tile_ld<DT>(base, rb + c, lane, x);
    acc8(op, A, x, K);
  }
  for (c += (long long)lane * 8; c < hi; c += EW_TILE) {
    float x[8];
    ld8<DT>(base, rb + c, x);
    acc8(op, A, x, K);
  }
}

// Columns [c0, c1) of a row starting at element rb of base split as
// [c0, ca) | [ca, cb) | [cb, c1), the middle 16-byte aligned and a multiple of
// 8 elements long (head and tail shorter than 8).
struct RowSplit {
  long long ca, cb;
};
template <int DT>
__device__ __forceinline__ RowSplit row_split(u64 base, long long rb, long long c0, long long c1) {
  constexpr int esz = DT == 0 ? 4 : 2;
  const u64 a = base + (u64)(rb + c0) * esz;
  long long head = (long long)(((16u - (unsigned)(a & 15)) & 15u) / esz);
  if (head > c1 - c0) head = c1 - c0;
  const long long ca = c0 + head;
  return RowSplit{ca, ca + ((c1 - ca) / 8) * 8};
}

template <int DT>
__device__ __forceinline__ float row_apply1(const RingEntry& E, int op, float p0, float p1, float x, long long c) {
  if (op == GPUOS_OP_SOFTMAX) return __fmul_rn(sm_exp(x - p0), p1);
  if (op == GPUOS_OP_RMSNORM) return __fmul_rn(__fmul_rn(x, p0), ld1<DT>(E.in1, c));
  return __fmaf_rn(__fmul_rn(x - p0, p1), ld1<DT>(E.in1, c), ld1<DT>(E.in2, c));
}

// Writes the outputs of columns [lo, hi) (same alignment rule as acc_span):
// input row, weights and output read and written in one layout.
template <int DT, int OP>
__device__ __forceinline__ void out_span(const RingEntry& E, float p0, float p1, long long rb, long long lo,
                                         long long hi, int lane) {
  long long c = lo;
  for (; c + EW_TILE <= hi; c += EW_TILE) {
    float x[8], w[8], b[8], y[8];
    tile_ld<DT>(E.in0, rb + c, lane, x);
    if (OP != GPUOS_OP_SOFTMAX) tile_ld<DT>(E.in1, c, lane, w);
    if (OP == GPUOS_OP_LAYERNORM) tile_ld<DT>(E.in2, c, lane, b);
    row_apply8(OP, p0, p1, x, w, b, y);
    tile_st<DT>(E.out, rb + c, lane, y);
  }
  for (c += (long long)lane * 8; c < hi; c += EW_TILE) {
    float x[8], w[8], b[8], y[8];
    ld8<DT>(E.in0, rb + c, x);
    if (OP != GPUOS_OP_SOFTMAX) ld8<DT>(E.in1, c, w);
    if (OP == GPUOS_OP_LAYERNORM) ld8<DT>(E.in2, c, b);
    row_apply8(OP, p0, p1, x, w, b, y);
    st8<DT>(E.out, rb + c, y);
  }
}

template <int DT, int OP>
static __device__ __noinline__ void row_out(const RingEntry& E, int, long long rb, long long c0, long long c1, Acc A, float K,
                        bool vec, int lane) {
  constexpr int op = OP;
  const long long cols = E.cols;
  float p0, p1;  // per-row constants
  row_consts(op, A, K, cols, E.s[0], p0, p1);
  if (vec) {
    out_span<DT, OP>(E, p0, p1, rb, c0, c1, lane);
  } else {
    // Unaligned row start. When the output (and the weights) sit at the same
    // offset modulo 16 bytes as the input row, the middle goes as ld8/st8.
    constexpr long long esz = DT == 0 ? 4 : 2;
    const RowSplit sp = row_split<DT>(E.in0, rb, c0, c1);
    const u64 shift = E.in0 + (u64)(rb * esz);
    bool pv = ((E.out - E.in0) & 15ull) == 0;
    if (op != GPUOS_OP_SOFTMAX) pv = pv && ((E.in1 - shift) & 15ull) == 0;
    if (op == GPUOS_OP_LAYERNORM) pv = pv && ((E.in2 - shift) & 15ull) == 0;
    if (pv) {
      if (lane < sp.ca - c0) {
        const long long c = c0 + lane;
        st1<DT>(E.out, rb + c, row_apply1<DT>(E, op, p0, p1, ld1<DT>(E.in0, rb + c), c));
      }
      if (lane < c1 - sp.cb) {
        const long long c = sp.cb + lane;
        st1<DT>(E.out, rb + c, row_apply1<DT>(E, op, p0, p1, ld1<DT>(E.in0, rb + c), c));
      }
      out_span<DT, OP>(E, p0, p1, rb, sp.ca, sp.cb, lane);
    } else {
      // Element at a time, eight loads issued before the first store.
      long long c = c0 + lane;
      for (; c + 7 * 32 < c1; c += 256) {
        float x[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = ld1<DT>(E.in0, rb + c + 32 * j);
#pragma unroll
        for (int j = 0; j < 8; ++j) st1<DT>(E.out, rb + c + 32 * j, row_apply1<DT>(E, op, p0, p1, x[j], c + 32 * j));
      }
      for (; c < c1; c += 32) st1<DT>(E.out, rb + c, row_apply1<DT>(E, op, p0, p1, ld1<DT>(E.in0, rb + c), c));
    }
  }
}

constexpr int ROW_UNR = 8;

// ------------------------------------------------------------------ staged row ops
// Statistic of ne elements (a multiple of 8) staged at shared address a.
template <int DT>
__device__ __forceinline__ void acc_s(int op, Acc& A, unsigned a, int ne, float K, int lane) {
  constexpr int ES = DT == 0 ? 4 : 2;
  for (int v = lane; v * 8 < ne; v += 32) {
    float x[8];
    lds8<DT>(a + (unsigned)(v * 8 * ES), x);
    acc8(op, A, x, K);
  }
}

// Output pass of ne staged elements: x at xa, weights at wa / ba (norms), to global element go.
template <int DT>
__device__ __forceinline__ void row_out_s(const RingEntry& E, int op, unsigned xa, unsigned wa, unsigned ba,
                                          long long go, int ne, float p0, float p1, int lane) {
  constexpr int ES = DT == 0 ? 4 : 2;
  for (int v = lane; v * 8 < ne; v += 32) {
    float x[8], w[8], b[8], y[8];
    lds8<DT>(xa + (unsigned)(v * 8 * ES), x);
    if (op == GPUOS_OP_RMSNORM || op == GPUOS_OP_LAYERNORM) lds8<DT>(wa + (unsigned)(v * 8 * ES), w);
    if (op == GPUOS_OP_LAYERNORM) lds8<DT>(ba + (unsigned)(v * 8 * ES), b);
    row_apply8(op, p0, p1, x, w, b, y);
    st8<DT>(E.out, go + v * 8, y);
  }
}

// Row item with every row segment staged through this warp's staging area by
// bulk copies: one copy brings a segment (and its weights), both passes read
// shared memory. Segments up to 4 KB (with weights) are pipelined three deep;
// up to 12 KB they use the whole area; longer segments stream in 4 KB chunks
// (read twice by two-pass ops, weights then from global memory). Requires
// 16-byte aligned tensors and cols % 8 == 0.
template <int DT, int OP>
static __device__ __noinline__ void row_staged(const RingEntry& E, u32 item, u32 row_chunk, const Cx cx) {
  constexpr int ES = DT == 0 ? 4 : 2;
  const long long rows = E.rows, cols = E.cols;
  const long long rpi = rows_per_item(cols, row_chunk);
  const long long r0 = (long long)item * rpi;
  const int R = (int)min(rpi, rows - r0);
  constexpr int op = OP;
  int S = 1;
  while (2 * S * R <= cx.nwarps && cols >= 512ll * S) S *= 2;  // cols / (2S) >= 256, without a division
  const int lgS = __ffs(S) - 1;                                     // S is a power of two
  long long seg = (cols + S - 1) >> lgS;
  seg = (seg + 7) & ~7ll;
  const int tasks = R * S;
  const int nwv = op == GPUOS_OP_RMSNORM ? 1 : (op == GPUOS_OP_LAYERNORM ? 2 : 0);
  const bool stats_only = (op == GPUOS_OP_ROWSUM || op == GPUOS_OP_ROWMAX);
  const long long unitb = seg * ES * (1 + nwv);
  const int mode = unitb <= WS_STAGE_BYTES ? 0 : (unitb <= WS_BYTES ? 1 : 2);
  const int lane = cx.lane, w = cx.warp, NW = cx.nwarps;
  const int mine = tasks > w ? (tasks - w + NW - 1) / NW : 0;
  const unsigned base = cx.ws->seq;
  unsigned u = base;  // next stage use
  __syncwarp();
  const unsigned char* in0 = reinterpret_cast<const unsigned char*>(E.in0);
  const unsigned char* in1 = reinterpret_cast<const unsigned char*>(E.in1);
  const unsigned char* in2 = reinterpret_cast<const unsigned char*>(E.in2);

  if (mode <= 1) {
    // one stage use per task; mode 0 keeps three tasks in flight
    auto issue = [&](int i) {  // lane 0
      const int t = w + i * NW;
      const int row = t >> lgS, sg = t & (S - 1);
      const long long c0 = (long long)sg * seg, c1 = min(cols, c0 + seg);
      const unsigned xb = (unsigned)((c1 - c0) * ES);
      const unsigned uu = base + (unsigned)i;
      unsigned long long* b = &cx.ws->bar[uu % WS_STAGES];
      unsigned char* dst = cx.ws->buf + (mode == 0 ? (uu % WS_STAGES) * WS_STAGE_BYTES : 0);
      mbar_arrive_expect_tx(b, xb * (unsigned)(1 + nwv));
      bulk_g2s(dst, in0 + ((r0 + row) * cols + c0) * ES, xb, b);
      if (nwv >= 1) bulk_g2s(dst + xb, in1 + c0 * ES, xb, b);
      if (nwv >= 2) bulk_g2s(dst + 2 * xb, in2 + c0 * ES, xb, b);
    };
    const int depth = mode == 0 ? WS_STAGES : 1;
    if (lane == 0) {
      fence_proxy_async_global();
      for (int i = 0; i < mine && i < depth; ++i) issue(i);
    }
    for (int i = 0; i < mine; ++i) {
      const int t = w + i * NW;
      const int row = t >> lgS, sg = t & (S - 1);
      const long long c0 = (long long)sg * seg, c1 = min(cols, c0 + seg);
      const int ne = (int)(c1 - c0);
      const unsigned uu = base + (unsigned)i;
      const unsigned xa = ws_addr(cx, mode == 0 ? (uu % WS_STAGES) * WS_STAGE_BYTES : 0);
      const unsigned wa = xa + (unsigned)(ne * ES), ba = xa + 2u * (unsigned)(ne * ES);
      const float K = op == GPUOS_OP_LAYERNORM ? ld1<DT>(E.in0, (r0 + row) * cols) : 0.f;
      ws_wait(cx, uu);
      Acc A = acc_init(op);
      acc_s<DT>(op, A, xa, ne, K, lane);
      acc_warp(op, A);
      if (S == 1) {
        if (stats_only) {
          if (lane == 0) st1<DT>(E.out, r0 + row, A.a);
        } else {
          float p0, p1;
          row_consts(op, A, K, cols, E.s[0], p0, p1);
          row_out_s<DT>(E, op, xa, wa, ba, (r0 + row) * cols + c0, ne, p0, p1, lane);
        }
      } else if (lane == 0) {
        cx.part[t] = make_float4(A.a, A.b, K, 0.f);
      }
      __syncwarp();
      if (lane == 0 && i + depth < mine) issue(i + depth);
    }
    u = base + (unsigned)mine;
    if (S > 1) {  // at most one task per warp here; its segment is still staged
      cx_sync(cx);
      if (mine == 1) {
        const int t = w;
        const int row = t >> lgS, sg = t & (S - 1);
        const long long c0 = (long long)sg * seg, c1 = min(cols, c0 + seg);
        const int ne = (int)(c1 - c0);
        const float4 q0 = cx.part[row * S];
        Acc A{q0.x, q0.y};
        const float K = q0.z;
        for (int j = 1; j < S; ++j) {
          const float4 q = cx.part[row * S + j];
          acc_merge(op, A, Acc{q.x, q.y});
        }
        if (stats_only) {
          if (sg == 0 && lane == 0) st1<DT>(E.out, r0 + row, A.a);
        } else {
          const unsigned xa = ws_addr(cx, mode == 0 ? (base % WS_STAGES) * WS_STAGE_BYTES : 0);
          float p0, p1;
          row_consts(op, A, K, cols, E.s[0], p0, p1);
          row_out_s<DT>(E, op, xa, xa + (unsigned)(ne * ES), xa + 2u * (unsigned)(ne * ES), (r0 + row) * cols + c0,
                        ne, p0, p1, lane);
        }
      }
    }
  } else {
    // long segments: stream x in 4 KB chunks through the three stages
    constexpr long long CHE = WS_STAGE_BYTES / ES;  // elements per chunk
    auto issue_chunk = [&](unsigned uu, long long gel, unsigned bytes) {  // lane 0
      unsigned long long* b = &cx.ws->bar[uu % WS_STAGES];
      mbar_arrive_expect_tx(b, bytes);
      bulk_g2s(cx.ws->buf + (uu % WS_STAGES) * WS_STAGE_BYTES, in0 + gel * ES, bytes, b);
    };
    // streams segment [gs, gs + ne) once; pass 0 accumulates, pass 1 writes outputs
    auto stream_pass = [&](long long gs, long long ne, int pass, Acc& A, float K, float p0, float p1,
                           long long cbase) {
      const int nch = (int)((ne + CHE - 1) / CHE);
      const unsigned ub = u;
      if (lane == 0) {
        fence_proxy_async_global();
        for (int k = 0; k < nch && k < WS_STAGES; ++k)
          issue_chunk(ub + (unsigned)k, gs + k * CHE, (unsigned)(min(CHE, ne - k * CHE) * ES));
      }
      for (int k = 0; k < nch; ++k) {
        const unsigned uu = ub + (unsigned)k;
        const int ce = (int)min(CHE, ne - k * CHE);
        ws_wait(cx, uu);
        const unsigned xa = ws_addr(cx, (uu % WS_STAGES) * WS_STAGE_BYTES);
        if (pass == 0) {
          acc_s<DT>(op, A, xa, ce, K, lane);
        } else {
          for (int v = lane; v * 8 < ce; v += 32) {
            float x[8], wv[8], bv[8], y[8];
            lds8<DT>(xa + (unsigned)(v * 8 * ES), x);
            const long long c = cbase + k * CHE + v * 8;  // column
            if (op == GPUOS_OP_RMSNORM || op == GPUOS_OP_LAYERNORM) ld8<DT>(E.in1, c, wv);
            if (op == GPUOS_OP_LAYERNORM) ld8<DT>(E.in2, c, bv);
            row_apply8(op, p0, p1, x, wv, bv, y);
            st8<DT>(E.out, gs + k * CHE + v * 8, y);
          }
        }
        __syncwarp();
        if (lane == 0 && k + WS_STAGES < nch)
          issue_chunk(ub + (unsigned)(k + WS_STAGES), gs + (k + WS_STAGES) * CHE,
                      (unsigned)(min(CHE, ne - (k + WS_STAGES) * CHE) * ES));
      }
      u = ub + (unsigned)nch;
    };
    for (int i = 0; i < mine; ++i) {
      const int t = w + i * NW;
      const int row = t >> lgS, sg = t & (S - 1);
      const long long c0 = (long long)sg * seg, c1 = min(cols, c0 + seg);
      const long long gs = (r0 + row) * cols + c0;
      const float K = op == GPUOS_OP_LAYERNORM ? ld1<DT>(E.in0, (r0 + row) * cols) : 0.f;
      Acc A = acc_init(op);
      stream_pass(gs, c1 - c0, 0, A, K, 0.f, 0.f, c0);
      acc_warp(op, A);
      if (S == 1) {
        if (stats_only) {
          if (lane == 0) st1<DT>(E.out, r0 + row, A.a);
        } else {
          float p0, p1;
          row_consts(op, A, K, cols, E.s[0], p0, p1);
          stream_pass(gs, c1 - c0, 1, A, K, p0, p1, c0);
        }
      } else if (lane == 0) {
        cx.part[t] = make_float4(A.a, A.b, K, 0.f);
      }
    }
    if (S > 1) {
      cx_sync(cx);
      if (mine == 1) {
        const int t = w;
        const int row = t >> lgS, sg = t & (S - 1);
        const long long c0 = (long long)sg * seg, c1 = min(cols, c0 + seg);
        const float4 q0 = cx.part[row * S];
        Acc A{q0.x, q0.y};
        const float K = q0.z;
        for (int j = 1; j < S; ++j) {
          const float4 q = cx.part[row * S + j];
          acc_merge(op, A, Acc{q.x, q.y});
        }
        if (stats_only) {
          if (sg == 0 && lane == 0) st1<DT>(E.out, r0 + row, A.a);
        } else {
          float p0, p1;
          row_consts(op, A, K, cols, E.s[0], p0, p1);
          stream_pass((r0 + row) * cols + c0, c1 - c0, 1, A, K, p0, p1, c0);
        }
      }
    }
  }
  if (lane == 0) cx.ws->seq = u % (2 * WS_STAGES);
  __syncwarp();
}

// cos and sin of pos * base^(-2i/cols), in double.
static __device__ __noinline__ double2 rotary_cs(double base, long long i, long long cols, int pos) {
  const double theta = pow(base, (-2.0 * (double)i) / (double)cols);
  const double phi = (double)pos * theta;
  double sn, cs;
  sincos(phi, &sn, &cs);
  return make_double2(cs, sn);
}

template <int DT>
static __device__ __noinline__ void rotary_item(const RingEntry& E, long long r0, int R, const Cx cx) {
  const long long cols = E.cols, half = cols / 2;
  const long long total = (long long)R * half;
  const double base = (double)E.s[0];
  long long ti = -1;  // the column pair whose angle is in cs, sn
  double cs = 0.0, sn = 0.0;
  const bool narrow = total <= 0x7fffffffll;  // 32-bit index arithmetic
  RotCache* rc = (cx.rot != nullptr && half <= ROT_MAX_PAIRS) ? cx.rot : nullptr;
  if (rc) {
    const bool hit = rc->cols == cols && rc->pos == E.pos && rc->base == E.s[0];
    if (!hit) {
      for (long long i = cx.tid; i < half; i += cx.nthr) rc->cs[i] = rotary_cs(base, i, cols, E.pos);
      cx_sync(cx);
      if (cx.tid == 0) {  // read by the next rotary op, after this item's closing barrier
        rc->cols = cols;
        rc->pos = E.pos;
        rc->base = E.s[0];
      }
    }
  }
  for (long long p = cx.tid; p < total; p += cx.nthr) {
    const long long row = narrow ? (long long)((u32)p / (u32)half) : p / half;
    const long long i = narrow ? (long long)((u32)p % (u32)half) : p % half;
    if (i != ti) {  // the angle depends on the column pair only
      const double2 t = rc ? rc->cs[i] : rotary_cs(base, i, cols, E.pos);
      cs = t.x;
      sn = t.y;
      ti = i;
    }
    const long long rb = (r0 + row) * cols;
    const double x1 = (double)ld1<DT>(E.in0, rb + i), x2 = (double)ld1<DT>(E.in0, rb + i + half);
    st1<DT>(E.out, rb + i, (float)(x1 * cs - x2 * sn));
    st1<DT>(E.out, rb + i + half, (float)(x2 * cs + x1 * sn));
  }
}

template <int DT, int OP>
static __device__ __noinline__ void row_item(const RingEntry& E, u32 item, u32 row_chunk, const Cx cx) {
  const long long rows = E.rows, cols = E.cols;
  const long long rpi = rows_per_item(cols, row_chunk);
  const long long r0 = (long long)item * rpi;
  const int R = (int)min(rpi, rows - r0);
  constexpr int op = OP;
  if constexpr (op == GPUOS_OP_ROTARY) {
    rotary_item<DT>(E, r0, R, cx);
    return;
  }
  int S = 1;  // warps per row
  while (2 * S * R <= cx.nwarps && cols >= 512ll * S) S *= 2;  // cols / (2S) >= 256, without a division
  const int lgS = __ffs(S) - 1;                                     // S is a power of two
  long long seg = (cols + S - 1) >> lgS;
  seg = (seg + 7) & ~7ll;
  const int tasks = R * S;
  bool vec = al16(E.in0) && (cols % 8) == 0;
  if (op == GPUOS_OP_SOFTMAX || op == GPUOS_OP_RMSNORM || op == GPUOS_OP_LAYERNORM) vec = vec && al16(E.out);
  if (op == GPUOS_OP_RMSNORM || op == GPUOS_OP_LAYERNORM) vec = vec && al16(E.in1);
  if (op == GPUOS_OP_LAYERNORM) vec = vec && al16(E.in2);
  const bool stats_only = (op == GPUOS_OP_ROWSUM || op == GPUOS_OP_ROWMAX);

  for (int t = cx.warp; t < tasks; t += cx.nwarps) {
    const int row = t >> lgS, sg = t & (S - 1);
    const long long c0 = (long long)sg * seg, c1 = min(cols, c0 + seg);
    const long long rb = (r0 + row) * cols;
    const float K = (op == GPUOS_OP_LAYERNORM) ? ld1<DT>(E.in0, rb) : 0.f;
    Acc A = acc_init(op);
    if (vec) {
      acc_span<DT, ROW_UNR>(op, A, K, E.in0, rb, c0, c1, cx.lane);
    } else {
      // Row start not 16-byte aligned (ragged lengths): the lanes take the
      // few head and tail elements one each, the aligned middle as ld8.
      const RowSplit sp = row_split<DT>(E.in0, rb, c0, c1);
      if (cx.lane < sp.ca - c0) acc1(op, A, ld1<DT>(E.in0, rb + c0 + cx.lane), K);
      if (cx.lane < c1 - sp.cb) acc1(op, A, ld1<DT>(E.in0, rb + sp.cb + cx.lane), K);
      acc_span<DT, ROW_UNR / 2>(op, A, K, E.in0, rb, sp.ca, sp.cb, cx.lane);
    }
    acc_warp(op, A);
    if (S == 1) {
      if (stats_only) {
        if (cx.lane == 0) st1<DT>(E.out, r0 + row, A.a);
      } else {
        row_out<DT, OP>(E, op, rb, 0, cols, A, K, vec, cx.lane);
      }
    } else if (cx.lane == 0) {
      cx.part[t] = make_float4(A.a, A.b, K, 0.f);
    }
  }
  if (S > 1) {
    cx_sync(cx);
    for (int t = cx.warp; t < tasks; t += cx.nwarps) {
      const int row = t >> lgS, sg = t & (S - 1);
      const long long c0 = (long long)sg * seg, c1 = min(cols, c0 + seg);
      const long long rb = (r0 + row) * cols;
      const float4 q0 = cx.part[row * S];
      Acc A{q0.x, q0.y};
      const float K = q0.z;
      for (int j = 1; j < S; ++j) {
        const float4 q = cx.part[row * S + j];
        acc_merge(op, A, Acc{q.x, q.y});
      }
      if (stats_only) {
        if (sg == 0 && cx.lane == 0) st1<DT>(E.out, r0 + row, A.a);
      } else {
        row_out<DT, OP>(E, op, rb, c0, c1, A, K, vec, cx.lane);
      }
    }
  }
}

// ------------------------------------------------------------------ dispatch
__device__ __forceinline__ void stall_item(const OpEnv& env, const Cx& cx) {
  if (cx.tid != 0 || env.st == nullptr) return;
  const u64 t0 = globaltimer();
  for (;;) {
    if (ld_relaxed_sys(&env.hctl->stall_gate) != 0) break;
    if (ld_relaxed_gpu(&env.st->abort_.v) != 0) break;
    if (globaltimer() - t0 > env.timeout_ns) {
      raise_error(env.st, env.hctl, GPUOS_ETIMEDOUT, env.id);
      break;
    }
    __nanosleep(1000);
  }
}

// Row bodies are instantiated per opcode so that each holds one op's code.
template <int DT, int OP>
__device__ __forceinline__ void row_one(const RingEntry& E, u32 item, u32 row_chunk, const Cx& cx, bool staged) {
  if (staged)
    row_staged<DT, OP>(E, item, row_chunk, cx);
  else
    row_item<DT, OP>(E, item, row_chunk, cx);
}
template <int DT>
__device__ __forceinline__ void row_dispatch(const RingEntry& E, u32 item, u32 row_chunk, const Cx& cx, bool staged) {
  switch (E.opcode) {
    case GPUOS_OP_ROWSUM: row_one<DT, GPUOS_OP_ROWSUM>(E, item, row_chunk, cx, staged); break;
    case GPUOS_OP_ROWMAX: row_one<DT, GPUOS_OP_ROWMAX>(E, item, row_chunk, cx, staged); break;
    case GPUOS_OP_SOFTMAX: row_one<DT, GPUOS_OP_SOFTMAX>(E, item, row_chunk, cx, staged); break;
    case GPUOS_OP_RMSNORM: row_one<DT, GPUOS_OP_RMSNORM>(E, item, row_chunk, cx, staged); break;
    case GPUOS_OP_LAYERNORM: row_one<DT, GPUOS_OP_LAYERNORM>(E, item, row_chunk, cx, staged); break;
    default: row_item<DT, GPUOS_OP_ROTARY>(E, item, row_chunk, cx); break;
  }
}

__device__ __forceinline__ void run_item(const RingEntry& E, u32 item, u32 elem_chunk, u32 row_chunk, const Cx& cx,
                                         const OpEnv& env) {
  const int op = E.opcode;
  if (op == GPUOS_OP_NOP) return;
  if (E.dtype <= 1) {
    if (op_is_ew(op)) {
      if (E.dtype == 0)
        ew_item<0>(E, item, elem_chunk, cx);
      else
        ew_item<1>(E, item, elem_chunk, cx);
      return;
    }
    if (op_is_row(op)) {
      bool staged = op != GPUOS_OP_ROTARY && al16(E.in0) && (E.cols % 8) == 0 && !(cx.flags & KF_NO_BULK);
      if (op == GPUOS_OP_SOFTMAX || op == GPUOS_OP_RMSNORM || op == GPUOS_OP_LAYERNORM) staged = staged && al16(E.out);
      if (op == GPUOS_OP_RMSNORM || op == GPUOS_OP_LAYERNORM) staged = staged && al16(E.in1);
      if (op == GPUOS_OP_LAYERNORM) staged = staged && al16(E.in2);
      if (E.dtype == 0)
        row_dispatch<0>(E, item, row_chunk, cx, staged);
      else
        row_dispatch<1>(E, item, row_chunk, cx, staged);
      return;
    }
  }
  if (op == GPUOS_OP_STALL) {
    stall_item(env, cx);
    return;
  }
  if (cx.tid == 0) raise_error(env.st, env.hctl, GPUOS_EBADOP, env.id);
}

}  // namespace gpuos_impl
