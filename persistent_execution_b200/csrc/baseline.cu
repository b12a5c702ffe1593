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

__global__ void __launch_bounds__(NCW * 32) gpuos_op_kernel(const RingEntry e, u32 elem_chunk, u32 row_chunk) {
  __shared__ RingEntry E;
  __shared__ float4 part[NCW];
  if (threadIdx.x < 8) reinterpret_cast<uint4*>(&E)[threadIdx.x] = reinterpret_cast<const uint4*>(&e)[threadIdx.x];
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
  const OpEnv env{nullptr, nullptr, 0ull, 0ull};
  for (u64 it = blockIdx.x; it < n; it += gridDim.x) {
    run_item(E, (u32)it, elem_chunk, row_chunk, cx, env);
    cx_sync(cx);
  }
}

void* op_kernel_fn() { return reinterpret_cast<void*>(&gpuos_op_kernel); }

void op_launch_dims(const RingEntry& e, u32 elem_chunk, u32 row_chunk, u32 sms, u32* grid, u32* block) {
  const u64 n = op_items(e.opcode, e.rows, e.cols, elem_chunk, row_chunk);
  const u64 cap = 4ull * sms;  // 4 CTAs of 512 threads fit on an SM
  *grid = (u32)(n < cap ? (n ? n : 1) : cap);
  *block = NCW * 32;
}

int launch_op(const RingEntry& e, u32 elem_chunk, u32 row_chunk, u32 sms, void* stream) {
  u32 g, b;
  op_launch_dims(e, elem_chunk, row_chunk, sms, &g, &b);
  gpuos_op_kernel<<<g, b, 0, static_cast<cudaStream_t>(stream)>>>(e, elem_chunk, row_chunk);
  return (int)cudaGetLastError();
}

}  // namespace gpuos_impl
