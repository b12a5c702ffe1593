// static_run.cu -- gpuos_run_static: one drained session of the persistent
// kernel whose scratch memory is a fixed array in the library's device image.
//
// Some callers must not allocate: cudaMalloc, cudaHostAlloc and cudaFree can
// block the whole device for milliseconds and can fail when another allocator
// (PyTorch's caching allocator, for example) already holds the memory. This
// entry point lets such callers run a batch of ops with no allocation at all:
// the descriptor ring, completion words, item counters and scheduler state
// live in g_scratch below, which every GPU that loads the library holds until
// the process exits.
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstring>

#include "internal.h"

using namespace gpuos_impl;

namespace {

constexpr u64 STATIC_MAX_OPS = 4096;   // ring entries; the limit on n
constexpr u32 STATIC_MAX_CTAS = 256;

// Byte offsets inside the scratch array.
constexpr size_t OFF_STATE = 0;
constexpr size_t OFF_CTL = 2048;
constexpr size_t OFF_RING = 4096;
constexpr size_t OFF_DONE = OFF_RING + STATIC_MAX_OPS * sizeof(RingEntry);
constexpr size_t OFF_HDONE = OFF_DONE + STATIC_MAX_OPS * sizeof(u64);
constexpr size_t OFF_TILES = OFF_HDONE + STATIC_MAX_OPS * sizeof(u64);
constexpr size_t OFF_STATS = OFF_TILES + STATIC_MAX_OPS * sizeof(u32);
constexpr size_t SCRATCH_BYTES = OFF_STATS + STATIC_MAX_CTAS * sizeof(CtaStats);
static_assert(sizeof(DevState) <= OFF_CTL, "state fits");
static_assert(sizeof(HostCtl) <= OFF_RING - OFF_CTL, "control block fits");

}  // namespace

// The scratch memory of gpuos_run_static (about 620 KB per device).
static __device__ __align__(256) unsigned char g_scratch[SCRATCH_BYTES];

namespace {

// Device address of g_scratch, looked up once per device with that device current.
constexpr int MAX_DEVICES = 64;
std::atomic<unsigned char*> g_scratch_ptr[MAX_DEVICES];

unsigned char* scratch_for(int dev) {
  if (dev < 0 || dev >= MAX_DEVICES) return nullptr;
  unsigned char* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  void* q = nullptr;
  if (cudaGetSymbolAddress(&q, g_scratch) != cudaSuccess || q == nullptr) {
    cudaGetLastError();
    return nullptr;
  }
  g_scratch_ptr[dev].store(static_cast<unsigned char*>(q), std::memory_order_release);
  return static_cast<unsigned char*>(q);
}

}  // namespace

extern "C" gpuos_status gpuos_run_static(const gpuos_desc* descs, uint64_t n, const gpuos_config* cfg_in,
                                         gpuos_stream_t stream) {
  if (!descs && n) return GPUOS_EINVAL;
  if (n > STATIC_MAX_OPS) return GPUOS_EINVAL;  // larger batches need gpuos_create's ring
  if (n == 0) return GPUOS_OK;
  gpuos_config cfg;
  if (cfg_in) {
    cfg = *cfg_in;
  } else if (gpuos_default_config(&cfg) != GPUOS_OK) {
    return GPUOS_EINVAL;
  }
  if (cfg.elem_chunk < 1024 || cfg.elem_chunk % 1024 != 0 || cfg.row_chunk < 1 || cfg.timeout_ns < 1000000ull ||
      cfg.idle_exit_ns < 1000000ull)
    return GPUOS_EINVAL;
  int dev = 0, sms = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
    return GPUOS_EDEVICE;
  const u32 grid = cfg.grid ? cfg.grid : (u32)sms;
  if (grid > STATIC_MAX_CTAS) return GPUOS_EINVAL;
  unsigned char* base = scratch_for(dev);
  if (!base) return GPUOS_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // Ring entries are built on the host in a small stack buffer and copied into
  // the scratch ring. Dependencies are indices into descs. Multi-item ops open
  // in submission order (prev_big), as in gpuos_submit.
  RingEntry buf[32];
  u64 last_big = 0;
  for (u64 i0 = 0; i0 < n; i0 += 32) {
    const u64 m = n - i0 < 32 ? n - i0 : 32;
    for (u64 j = 0; j < m; ++j) {
      const u64 id = i0 + j;
      const gpuos_desc* d = &descs[id];
      if (gpuos_validate(d) != GPUOS_OK || d->opcode == GPUOS_OP_STALL) return GPUOS_EINVAL;
      RingEntry& e = buf[j];
      std::memset(&e, 0, sizeof(e));
      const long long nel = d->rows * d->cols;
      e.in0 = (u64)d->in[0];
      e.in1 = (u64)d->in[1];
      e.in2 = (u64)d->in[2];
      e.out = (u64)d->out;
      e.rows = d->rows;
      e.cols = d->cols;
      if (op_is_ew(d->opcode)) {
        e.in_n0 = d->in_n[0] > 0 ? d->in_n[0] : nel;
        e.in_n1 = d->in_n[1] > 0 ? d->in_n[1] : nel;
      } else {
        e.in_n0 = nel;
        e.in_n1 = d->cols;
      }
      for (int k = 0; k < 4; ++k) e.s[k] = d->s[k];
      e.pos = d->pos;
      e.opcode = d->opcode;
      e.dtype = d->dtype;
      e.nmicro = d->nmicro;
      for (int k = 0; k < 8; ++k) e.micro[k] = d->micro[k];
      u64 dep[2];
      for (int k = 0; k < 2; ++k) {
        if (d->dep[k] == GPUOS_NO_DEP) {
          dep[k] = 0;
        } else {
          if (d->dep[k] >= id) return GPUOS_EINVAL;
          dep[k] = d->dep[k] + 1;
        }
      }
      e.dep0 = dep[0];
      e.dep1 = dep[1];
      const u64 items = (d->opcode == GPUOS_OP_NOP) ? 1 : op_items(d->opcode, d->rows, d->cols, cfg.elem_chunk, cfg.row_chunk);
      if (items == 0 || items > MAX_ITEMS) return GPUOS_EINVAL;
      if (items > 1) {
        e.prev_big = last_big;
        last_big = id + 1;
      }
      e.hdr = hdr_make(id, false, items);
    }
    if (cudaMemcpyAsync(base + OFF_RING + i0 * sizeof(RingEntry), buf, m * sizeof(RingEntry),
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
      return GPUOS_EDEVICE;
  }
  // Every call reuses the array: ids restart at 0, so the completion words,
  // item counters and the error word must start at zero.
  if (cudaMemsetAsync(base + OFF_DONE, 0, n * sizeof(u64), s) != cudaSuccess ||
      cudaMemsetAsync(base + OFF_CTL, 0, sizeof(HostCtl), s) != cudaSuccess)
    return GPUOS_EDEVICE;

  KParams p;
  p.st = reinterpret_cast<DevState*>(base + OFF_STATE);
  p.dring = reinterpret_cast<RingEntry*>(base + OFF_RING);
  p.done = reinterpret_cast<u64*>(base + OFF_DONE);
  p.tiles_done = reinterpret_cast<u32*>(base + OFF_TILES);
  p.hring = p.dring;  // the entries are already in place; the fetcher copies them onto themselves
  p.hctl = reinterpret_cast<HostCtl*>(base + OFF_CTL);
  p.hdone = reinterpret_cast<u64*>(base + OFF_HDONE);
  p.stats = reinterpret_cast<CtaStats*>(base + OFF_STATS);
  p.trace = nullptr;
  p.owner = nullptr;  // no chain hand-off: the array holds no mailboxes
  p.mbox = nullptr;
  p.mctl = nullptr;
  p.mask = STATIC_MAX_OPS - 1;
  p.base = 0;
  p.fetched_upto = 0;  // the fetchers copy the entries onto themselves
  p.timeout_ns = cfg.timeout_ns;
  p.idle_exit_ns = cfg.idle_exit_ns;
  p.elem_chunk = cfg.elem_chunk;
  p.row_chunk = cfg.row_chunk;
  p.backoff_ns = cfg.backoff_ns;
  p.flags = KF_DRAIN;
  p.grid = grid;
  if (launch_session(p, n, 0ull, s) != 0) return GPUOS_EDEVICE;
  unsigned int status = 0;
  if (cudaMemcpyAsync(&status, base + OFF_CTL + offsetof(HostCtl, status), sizeof(status), cudaMemcpyDeviceToHost,
                      s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return GPUOS_EDEVICE;
  return static_cast<gpuos_status>(status);
}
