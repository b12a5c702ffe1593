// baseline.cu -- one kernel launch per op, with the same op bodies as the
// persistent kernel ("Kernel Launch and Host-Device Interaction", section 5,
// "The launch path": every op pays the host launch steps 1-4 and the GPU
// front-end steps 5-6). The same launches, captured into a CUDA Graph, form
// the graph-replay baseline ("Launch Overhead and Fusion", section
// "Graph capture").
#include <cuda_runtime.h>

#include "internal.h"
#include "ops.cuh"

namespace gpuos_impl {

constexpr size_t OP_SMEM = NCW * sizeof(WarpSmem);  // one staging area per warp

__global__ void __launch_bounds__(NCW * 32) gpuos_op_kernel(const RingEntry e, u32 elem_chunk, u32 row_chunk) {
  __shared__ RingEntry E;
  __shared__ float4 part[NCW];
  extern __shared__ __align__(128) unsigned char dsm[];
  WarpSmem* W = reinterpret_cast<WarpSmem*>(dsm);
  if (threadIdx.x < 8) reinterpret_cast<uint4*>(&E)[threadIdx.x] = reinterpret_cast<const uint4*>(&e)[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int wi = 0; wi < (int)(blockDim.x >> 5); ++wi) {
      W[wi].seq = 0;
      for (int j = 0; j < WS_STAGES; ++j) mbar_init(&W[wi].bar[j], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const u64 n = op_items(E.opcode, E.rows, E.cols, elem_chunk, row_chunk);
  Cx cx;
  cx.tid = threadIdx.x;
  cx.nthr = blockDim.x;
  cx.warp = threadIdx.x >> 5;
  cx.nwarps = blockDim.x >> 5;
  cx.lane = threadIdx.x & 31;
  cx.bar = 1;
  cx.part = part;
  cx.ws = W + cx.warp;
  cx.st = nullptr;
  cx.hctl = nullptr;
  cx.id = 0;
  cx.flags = 0;
  cx.rot = nullptr;
  const OpEnv env{nullptr, nullptr, 0ull, 0ull};
  for (u64 it = blockIdx.x; it < n; it += gridDim.x) {
    run_item(E, (u32)it, elem_chunk, row_chunk, cx, env);
    cx_sync(cx);
  }
}

void* op_kernel_fn() { return reinterpret_cast<void*>(&gpuos_op_kernel); }

size_t op_smem_bytes() {
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(gpuos_op_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)OP_SMEM) == cudaSuccess)
      attr_set = true;
  }
  return OP_SMEM;
}

void op_launch_dims(const RingEntry& e, u32 elem_chunk, u32 row_chunk, u32 sms, u32* grid, u32* block) {
  const u64 n = op_items(e.opcode, e.rows, e.cols, elem_chunk, row_chunk);
  const u64 cap = 1ull * sms;  // one CTA per SM (its staging areas take most of shared memory)
  *grid = (u32)(n < cap ? (n ? n : 1) : cap);
  *block = NCW * 32;
}

int launch_op(const RingEntry& e, u32 elem_chunk, u32 row_chunk, u32 sms, void* stream) {
  u32 g, b;
  op_launch_dims(e, elem_chunk, row_chunk, sms, &g, &b);
  const size_t sm = op_smem_bytes();
  gpuos_op_kernel<<<g, b, sm, static_cast<cudaStream_t>(stream)>>>(e, elem_chunk, row_chunk);
  return (int)cudaGetLastError();
}

}  // namespace gpuos_impl
