// runtime.cu -- host side of the persistent op-queue runtime: the C ABI of
// include/gpuos.h.
//
// Submission path (no CUDA call per op): validate the descriptor, give it the
// next dense id, build its 128-byte ring entry and write it into the pinned,
// write-combined, device-mapped ring. Flush is a store fence plus one store of
// the head counter into mapped memory -- the user-space counterpart of the
// driver's pinned host ring and doorbell ("Kernel Launch and Host-Device
// Interaction", section 5, "The launch path").
// Waiting reads the per-op completion entries the device writes into mapped
// memory, so there is no implicit synchronisation per op (same page,
// "Synchronization primitives").
#include <cuda_runtime.h>
#include <immintrin.h>

#include <algorithm>
#include <chrono>
#include <cstring>
#include <deque>
#include <new>
#include <vector>

#include "internal.h"

using namespace gpuos_impl;

namespace {

u64 now_ns() {
  return (u64)std::chrono::duration_cast<std::chrono::nanoseconds>(
             std::chrono::steady_clock::now().time_since_epoch())
      .count();
}

const u64 MAX_ELEMS = 1ull << 40;

bool known_opcode(int op) {
  return op == GPUOS_OP_NOP || (op >= GPUOS_OP_ADD && op <= GPUOS_OP_EW_CHAIN) ||
         (op >= GPUOS_OP_ROWSUM && op <= GPUOS_OP_ROTARY) || op == GPUOS_OP_STALL;
}

void chain_uses(const gpuos_desc* d, bool* u1, bool* u2, int* nscal, bool* ok) {
  *u1 = *u2 = false;
  *nscal = 0;
  *ok = d->nmicro >= 1 && d->nmicro <= 8;
  for (int i = 0; *ok && i < d->nmicro; ++i) {
    const int m = d->micro[i];
    if (m < GPUOS_M_AFFINE || m > GPUOS_M_MUL2) *ok = false;
    if (m == GPUOS_M_AFFINE) *nscal += 2;
    if (m == GPUOS_M_SCALE || m == GPUOS_M_ADDS) *nscal += 1;
    if (m == GPUOS_M_ADD1 || m == GPUOS_M_MUL1) *u1 = true;
    if (m == GPUOS_M_ADD2 || m == GPUOS_M_MUL2) *u2 = true;
  }
  if (*nscal > 4) *ok = false;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

gpuos_status validate_desc(const gpuos_desc* d, const gpuos_config* cfg) {
  if (!d) return GPUOS_EINVAL;
  const int op = d->opcode;
  if (!known_opcode(op)) return GPUOS_EINVAL;
  if (d->dtype > GPUOS_BF16) return GPUOS_EINVAL;
  if (d->flags != 0 || d->reserved0 != 0 || d->reserved1 != 0) return GPUOS_EINVAL;
  if (op == GPUOS_OP_NOP || op == GPUOS_OP_STALL) return GPUOS_OK;
  if (d->rows < 1 || d->cols < 1) return GPUOS_EINVAL;
  if ((u64)d->rows > MAX_ELEMS || (u64)d->cols > MAX_ELEMS || (u64)d->rows > MAX_ELEMS / (u64)d->cols)
    return GPUOS_EINVAL;
  const size_t es = d->dtype == GPUOS_F32 ? 4 : 2;
  if (!d->out || !aligned(d->out, es) || !d->in[0] || !aligned(d->in[0], es)) return GPUOS_EINVAL;
  bool need1 = false, need2 = false;
  if (op == GPUOS_OP_ADD || op == GPUOS_OP_MUL || op == GPUOS_OP_SILU_MUL || op == GPUOS_OP_RMSNORM ||
      op == GPUOS_OP_LAYERNORM)
    need1 = true;
  if (op == GPUOS_OP_LAYERNORM) need2 = true;
  if (op == GPUOS_OP_EW_CHAIN) {
    int nsc;
    bool ok;
    chain_uses(d, &need1, &need2, &nsc, &ok);
    if (!ok) return GPUOS_EINVAL;
  }
  if (need1 && (!d->in[1] || !aligned(d->in[1], es))) return GPUOS_EINVAL;
  if (need2 && (!d->in[2] || !aligned(d->in[2], es))) return GPUOS_EINVAL;
  if (op_is_ew(op) && (d->in_n[0] < 0 || d->in_n[1] < 0)) return GPUOS_EINVAL;
  if (op == GPUOS_OP_ROTARY && (d->cols % 2) != 0) return GPUOS_EINVAL;
  const u64 items = op_items(op, d->rows, d->cols, cfg->elem_chunk, cfg->row_chunk);
  if (items == 0 || items > MAX_ITEMS) return GPUOS_EINVAL;
  return GPUOS_OK;
}

// Builds the ring entry of a validated descriptor (header and dependencies
// are filled in by the caller).
void build_entry(const gpuos_desc* d, const gpuos_config* cfg, RingEntry* e) {
  std::memset(e, 0, sizeof(*e));
  const long long n = d->rows * d->cols;
  e->in0 = (u64)d->in[0];
  e->in1 = (u64)d->in[1];
  e->in2 = (u64)d->in[2];
  e->out = (u64)d->out;
  e->rows = d->rows;
  e->cols = d->cols;
  if (op_is_ew(d->opcode)) {
    e->in_n0 = d->in_n[0] > 0 ? d->in_n[0] : n;
    e->in_n1 = d->in_n[1] > 0 ? d->in_n[1] : n;
  } else {
    e->in_n0 = n;
    e->in_n1 = d->cols;
  }
  for (int i = 0; i < 4; ++i) e->s[i] = d->s[i];
  e->pos = d->pos;
  e->opcode = d->opcode;
  e->dtype = d->dtype;
  e->nmicro = d->nmicro;
  for (int i = 0; i < 8; ++i) e->micro[i] = d->micro[i];
  (void)cfg;
}

void default_config(gpuos_config* c) {
  c->ring_capacity = 131072;
  c->grid = 0;
  c->timeout_ns = 2000000000ull;
  c->submit_timeout_ns = 2000000000ull;
  c->idle_exit_ns = 20000000000ull;
  c->elem_chunk = 262144;  // large ops: few, long items (fewer claims; the grid streams HBM)
  c->row_chunk = 524288;
  c->backoff_ns = 1000;
  c->flags = 0;
}

}  // namespace

struct gpuos {
  int dev = 0;
  cudaStream_t stream = nullptr;
  cudaStream_t aux = nullptr;
  gpuos_config cfg;
  u32 grid = 0, sms = 0;
  RingEntry* hring = nullptr;
  HostCtl* hctl = nullptr;
  u64* hdone = nullptr;
  RingEntry* hring_d = nullptr;
  HostCtl* hctl_d = nullptr;
  u64* hdone_d = nullptr;
  DevState* st = nullptr;
  RingEntry* dring = nullptr;
  u64* done = nullptr;
  u32* tiles_done = nullptr;
  u64* owner = nullptr;
  u64* mbox = nullptr;
  MailCtl* mctl = nullptr;
  CtaStats* cstats = nullptr;
  gpuos_trace_rec* trace = nullptr;
  u64 cap = 0, mask = 0;
  u64 next_id = 0, published = 0, tail = 0, session_base = 0;
  u64 dma_upto = 0;               // ids below this were copied into the device ring by the copy engine
  RingEntry last_e;               // entry of op next_id - 1 as written to the ring
  bool last_fusable = false;      // that op may head a fused pair
  cudaEvent_t dma_ev = nullptr;   // the last such copy
  bool running = false;
  bool kernel_alive = false;  // false only if a kernel could not be confirmed stopped
  u32 run_flags = 0;
  u64 run_head = 0;  // ops published when the running session started
  bool prev_single = false;
  u64 prev_chain_start = 0;
  u64 last_big = 0;  // id + 1
  std::deque<u64> big_ids;
  u64 retired_big = 0;  // id + 1
  gpuos_status sticky = GPUOS_OK;
  u64 err_op = 0;
  u64 max_occ = 0, launches = 0;
  u64 acc_items = 0, acc_claimed = 0, acc_run = 0, acc_idle = 0, acc_dep = 0, acc_fetch = 0;
  u64 last_span = 0;
};

namespace {

void refresh_tail(gpuos* rt) {
  while (rt->tail < rt->next_id) {
    const u64 v = __atomic_load_n(&rt->hdone[rt->tail & rt->mask], __ATOMIC_ACQUIRE);
    if (v != rt->tail + 1) break;
    ++rt->tail;
  }
  if (rt->sticky == GPUOS_OK) {
    const u32 s = __atomic_load_n(&rt->hctl->status, __ATOMIC_ACQUIRE);
    if (s != 0) {
      rt->sticky = (gpuos_status)s;
      rt->err_op = rt->hctl->err_id;
    }
  }
}

// Waits for the persistent kernel to leave after stop was requested (or it drained).
gpuos_status join_kernel(gpuos* rt, u64 timeout_ns) {
  const u64 t0 = now_ns();
  for (;;) {
    const cudaError_t q = cudaStreamQuery(rt->stream);
    if (q == cudaSuccess) break;
    if (q != cudaErrorNotReady) {
      rt->running = false;
      rt->sticky = GPUOS_EDEVICE;
      return GPUOS_EDEVICE;
    }
    if (now_ns() - t0 > timeout_ns) return GPUOS_EDEVICE;  // kernel still alive: keep memory
    _mm_pause();
  }
  rt->running = false;
  rt->kernel_alive = false;
  // fold the session's device counters into the totals
  std::vector<CtaStats> cs(rt->grid);
  DevState ds;
  if (cudaMemcpyAsync(cs.data(), rt->cstats, sizeof(CtaStats) * rt->grid, cudaMemcpyDeviceToHost, rt->aux) ==
          cudaSuccess &&
      cudaMemcpyAsync(&ds, rt->st, sizeof(DevState), cudaMemcpyDeviceToHost, rt->aux) == cudaSuccess &&
      cudaStreamSynchronize(rt->aux) == cudaSuccess) {
    for (const CtaStats& c : cs) {
      rt->acc_items += c.items;
      rt->acc_claimed += c.ops_claimed;
      rt->acc_run += c.run_ops;
      rt->acc_idle += c.idle_cycles;
      rt->acc_dep += c.dep_cycles;
      rt->acc_fetch += c.fetch_descs;
    }
    rt->last_span = ds.span_end.v > ds.span_start.v ? ds.span_end.v - ds.span_start.v : 0;
  }
  refresh_tail(rt);
  return GPUOS_OK;
}

void retire_bigs(gpuos* rt, u64 upto) {
  while (!rt->big_ids.empty() && rt->big_ids.front() < upto) {
    rt->retired_big = rt->big_ids.front() + 1;
    rt->big_ids.pop_front();
  }
}

// Copies the host entries of ids [from, to) into their device-ring slots with
// the copy engine (aux stream). A drained session then starts with its whole
// stream in device memory: its CTAs do not read descriptors over PCIe while
// ops run, which would hold up the loads of the running ops on every SM.
bool dma_ring(gpuos* rt, u64 from, u64 to) {
  while (from < to) {
    const u64 s = from & rt->mask;
    const u64 m = std::min(to - from, rt->cap - s);
    if (cudaMemcpyAsync(rt->dring + s, rt->hring + s, m * sizeof(RingEntry), cudaMemcpyHostToDevice, rt->aux) !=
        cudaSuccess)
      return false;
    from += m;
  }
  rt->dma_upto = to;
  return cudaEventRecord(rt->dma_ev, rt->aux) == cudaSuccess;
}

gpuos_status start_kernel(gpuos* rt, u32 flags) {
  if (rt->sticky != GPUOS_OK) return rt->sticky;
  if (rt->running) return GPUOS_EINVAL;
  refresh_tail(rt);
  const u64 base = rt->tail;
  retire_bigs(rt, base);
  const u64 big_init = rt->retired_big ? ((rt->retired_big << 24) | BIG_EXHAUSTED) : 0ull;
  rt->hctl->stop = 0;
  rt->hctl->exited_idle = 0;
  _mm_sfence();
  KParams p;
  p.st = rt->st;
  p.dring = rt->dring;
  p.done = rt->done;
  p.tiles_done = rt->tiles_done;
  p.hring = rt->hring_d;
  p.hctl = rt->hctl_d;
  p.hdone = rt->hdone_d;
  p.stats = rt->cstats;
  p.trace = rt->trace;
  const bool handoff = !(rt->cfg.flags & GPUOS_CFG_NO_HANDOFF);
  p.owner = handoff ? rt->owner : nullptr;
  p.mbox = handoff ? rt->mbox : nullptr;
  p.mctl = handoff ? rt->mctl : nullptr;
  p.mask = rt->mask;
  p.base = base;
  p.timeout_ns = rt->cfg.timeout_ns;
  p.idle_exit_ns = rt->cfg.idle_exit_ns;
  p.elem_chunk = rt->cfg.elem_chunk;
  p.row_chunk = rt->cfg.row_chunk;
  p.backoff_ns = rt->cfg.backoff_ns;
  p.flags = ((flags & GPUOS_START_DRAIN) ? KF_DRAIN : 0u) | ((rt->cfg.flags & GPUOS_CFG_TRACE) ? KF_TRACE : 0u) |
            ((rt->cfg.flags & GPUOS_CFG_NO_BULK) ? KF_NO_BULK : 0u);
  p.grid = rt->grid;
  // Entries of this session not yet in the device ring: copied now (drained
  // sessions) or fetched by the kernel (live sessions).
  if (flags & GPUOS_START_DRAIN) {
    const u64 from = std::max(rt->dma_upto, base);
    if (from < rt->published && !dma_ring(rt, from, rt->published)) {
      rt->sticky = GPUOS_EDEVICE;
      return GPUOS_EDEVICE;
    }
  }
  if (rt->dma_upto > base && cudaStreamWaitEvent(rt->stream, rt->dma_ev, 0) != cudaSuccess) {
    rt->sticky = GPUOS_EDEVICE;
    return GPUOS_EDEVICE;
  }
  p.fetched_upto = std::min(std::max(rt->dma_upto, base), rt->published);
  const int e = launch_session(p, rt->published, big_init, rt->stream);
  if (e != 0) {
    rt->sticky = GPUOS_EDEVICE;
    return GPUOS_EDEVICE;
  }
  rt->launches += 2;
  rt->running = true;
  rt->kernel_alive = true;
  rt->run_flags = flags;
  rt->run_head = rt->published;
  rt->session_base = base;
  return GPUOS_OK;
}

// Flushes of at least this many new ops to a live kernel are copied into the
// device ring by the copy engine before the head moves; smaller ones are
// fetched by the kernel's control warps.
constexpr u64 LIVE_DMA_MIN = 128;

gpuos_status publish(gpuos* rt) {
  _mm_sfence();
  const u64 old = rt->published;
  const bool live = rt->running && !(rt->run_flags & GPUOS_START_DRAIN);
  if (live && rt->next_id - old >= LIVE_DMA_MIN) {
    // Every entry of the session not yet copied goes now (entries the kernel
    // fetched itself are rewritten with the same bytes); the head moves only
    // after the copy completed, so the kernel never reads a partial entry.
    const u64 from = std::max(rt->dma_upto, rt->session_base);
    if (!dma_ring(rt, from, rt->next_id) || cudaEventSynchronize(rt->dma_ev) != cudaSuccess) {
      rt->sticky = GPUOS_EDEVICE;
      return GPUOS_EDEVICE;
    }
    __atomic_store_n(&rt->hctl->dma_head, rt->next_id, __ATOMIC_RELEASE);
  }
  __atomic_store_n(&rt->hctl->head, rt->next_id, __ATOMIC_RELEASE);
  rt->published = rt->next_id;
  // With no kernel running, or a drained one (which never reads ids at or
  // past its own head), the new entries go to the device ring right away.
  if (!rt->running || (rt->run_flags & GPUOS_START_DRAIN)) {
    const u64 from = std::max(rt->dma_upto, old);
    if (from < rt->published && !dma_ring(rt, from, rt->published)) {
      rt->sticky = GPUOS_EDEVICE;
      return GPUOS_EDEVICE;
    }
  }
  return GPUOS_OK;
}

gpuos_status flush_impl(gpuos* rt) {
  if (rt->sticky != GPUOS_OK) return rt->sticky;
  if (rt->running && !(rt->run_flags & GPUOS_START_DRAIN) &&
      __atomic_load_n(&rt->hctl->exited_idle, __ATOMIC_ACQUIRE)) {
    gpuos_status s = join_kernel(rt, 2 * rt->cfg.timeout_ns + 5000000000ull);
    if (s != GPUOS_OK) return s;
    publish(rt);
    return start_kernel(rt, 0);
  }
  return publish(rt);
}

gpuos_status wait_impl(gpuos* rt, u64 id, u64 timeout_ns) {
  refresh_tail(rt);
  if (rt->sticky != GPUOS_OK) return rt->sticky;
  u64 target;
  if (id == GPUOS_ALL) {
    if (rt->next_id == 0) return GPUOS_OK;
    target = rt->next_id - 1;
  } else {
    if (id >= rt->next_id) return GPUOS_EINVAL;
    target = id;
  }
  if (rt->tail > target) return GPUOS_OK;
  if (target >= rt->published) {
    gpuos_status s = flush_impl(rt);
    if (s != GPUOS_OK) return s;
  }
  const u64 t0 = now_ns();
  for (u32 it = 1;; ++it) {
    refresh_tail(rt);
    if (rt->tail > target) return GPUOS_OK;
    if (rt->sticky != GPUOS_OK) return rt->sticky;
    if ((it & 1023) == 0) {
      if (!rt->running) return GPUOS_ESTOPPED;
      if (cudaStreamQuery(rt->stream) != cudaErrorNotReady) {
        // the kernel left (drained, idled or failed); collect what completed
        join_kernel(rt, 1000000000ull);
        refresh_tail(rt);
        if (rt->tail > target) return GPUOS_OK;
        if (rt->sticky != GPUOS_OK) return rt->sticky;
        if (__atomic_load_n(&rt->hctl->exited_idle, __ATOMIC_ACQUIRE)) {
          gpuos_status s = start_kernel(rt, 0);
          if (s != GPUOS_OK) return s;
          continue;
        }
        return GPUOS_ESTOPPED;
      }
      if (now_ns() - t0 > timeout_ns) return GPUOS_ETIMEDOUT;
    }
    _mm_pause();
  }
}

// Fused pairs (NEXT step of the method: dynamic fusion of consecutive
// elementwise ops, GPUOS page, "The Paper" and "What's New"; "Launch Overhead
// and Fusion", "Fusion"). An fp32 single-item op whose program is scalar
// micro-ops only (relu-affine or a chain of affine/scale/adds/relu) can head a
// pair; the next op, if it is the same kind of op, reads the head's output as
// its direct first operand over the same elements and depends on the head
// alone, is folded into the head's entry while both are still unpublished.
// The program becomes head, M_STORE1, tail with in1 = the head's output: both
// outputs are written, bit-identical to running the two ops one after the
// other (each micro-op rounds to fp32 either way). The tail becomes a NOP that
// depends on the head, so completion order and dependants are unchanged.
int scalar_program(const RingEntry& e, unsigned char* prog, int* nscal) {
  if (e.opcode == GPUOS_OP_RELU_AFFINE) {
    prog[0] = GPUOS_M_AFFINE;
    prog[1] = GPUOS_M_RELU;
    *nscal = 2;
    return 2;
  }
  if (e.opcode != GPUOS_OP_EW_CHAIN) return -1;
  int k = 0;
  for (int i = 0; i < e.nmicro; ++i) {
    const int m = e.micro[i];
    if (m == GPUOS_M_AFFINE)
      k += 2;
    else if (m == GPUOS_M_SCALE || m == GPUOS_M_ADDS)
      k += 1;
    else if (m != GPUOS_M_RELU)
      return -1;
    prog[i] = (unsigned char)m;
  }
  *nscal = k;
  return e.nmicro;
}

bool fusable(const RingEntry& e, bool single) {
  unsigned char prog[8];
  int ns = 0;
  return single && e.dtype == GPUOS_F32 && e.in_n0 == e.rows * e.cols && scalar_program(e, prog, &ns) >= 0 &&
         ns <= 4;
}

// Folds entry b (op id) into the previous entry a; true if fused.
bool try_fuse(gpuos* rt, u64 id, RingEntry& a, const RingEntry& b) {
  if ((rt->cfg.flags & GPUOS_CFG_NO_FUSION) || !rt->last_fusable || id == 0 || id - 1 < rt->published) return false;
  if (b.in0 != a.out || b.rows * b.cols != a.rows * a.cols || b.in_n0 != a.rows * a.cols) return false;
  if (!((b.dep0 == id && b.dep1 == 0) || (b.dep1 == id && b.dep0 == 0))) return false;  // depends on id - 1 alone
  unsigned char pa[8], pb[8];
  int ka = 0, kb = 0;
  const int na = scalar_program(a, pa, &ka), nb = scalar_program(b, pb, &kb);
  if (na < 0 || nb < 0 || ka + kb > 4 || na + 1 + nb > 8) return false;
  RingEntry f = a;
  f.opcode = GPUOS_OP_EW_CHAIN;
  for (int i = 0; i < na; ++i) f.micro[i] = pa[i];
  f.micro[na] = M_STORE1;
  for (int i = 0; i < nb; ++i) f.micro[na + 1 + i] = pb[i];
  for (int i = na + 1 + nb; i < 8; ++i) f.micro[i] = 0;
  f.nmicro = (unsigned char)(na + 1 + nb);
  for (int i = 0; i < kb; ++i) f.s[ka + i] = b.s[i];
  f.in1 = a.out;
  f.in_n1 = a.rows * a.cols;
  f.out = b.out;
  a = f;
  return true;
}

void write_entry(gpuos* rt, u64 id, const RingEntry& e) {
  __m128i* dst = reinterpret_cast<__m128i*>(&rt->hring[id & rt->mask]);
  const __m128i* src = reinterpret_cast<const __m128i*>(&e);
  for (int j = 0; j < 8; ++j) _mm_stream_si128(dst + j, _mm_load_si128(src + j));
}

gpuos_status submit_one(gpuos* rt, const gpuos_desc* d, u64 dep_base, u64 first_id, u64* id_out, bool raw) {
  if (rt->sticky != GPUOS_OK) return rt->sticky;
  if (!raw) {
    const gpuos_status s = validate_desc(d, &rt->cfg);
    if (s != GPUOS_OK) return s;
  } else if (!d) {
    return GPUOS_EINVAL;
  }
  const u64 id = rt->next_id;
  u64 dep[2];
  for (int k = 0; k < 2; ++k) {
    u64 v = d->dep[k];
    if (v == GPUOS_NO_DEP) {
      dep[k] = 0;
      continue;
    }
    if (dep_base != GPUOS_NO_BASE) {  // caller numbering in which descs[0] is dep_base
      if (v + first_id < dep_base) return GPUOS_EINVAL;
      v = v + first_id - dep_base;
    }
    if (v >= id) return GPUOS_EINVAL;
    dep[k] = v + 1;
  }
  // ring space: slot id & mask is free once op id - cap completed
  if (id - rt->tail >= rt->cap) {
    refresh_tail(rt);
    if (id - rt->tail >= rt->cap) {
      if (!rt->running) return GPUOS_EAGAIN;
      gpuos_status s = flush_impl(rt);
      if (s != GPUOS_OK) return s;
      const u64 t0 = now_ns();
      while (id - rt->tail >= rt->cap) {
        refresh_tail(rt);
        if (rt->sticky != GPUOS_OK) return rt->sticky;
        if (now_ns() - t0 > rt->cfg.submit_timeout_ns) return GPUOS_EAGAIN;
        _mm_pause();
      }
    }
  }
  RingEntry e;
  build_entry(d, &rt->cfg, &e);
  u64 items = known_opcode(d->opcode) && d->rows > 0 && d->cols > 0
                  ? op_items(d->opcode, d->rows, d->cols, rt->cfg.elem_chunk, rt->cfg.row_chunk)
                  : 1;
  if (items == 0 || items > MAX_ITEMS) items = 1;
  const bool single = items == 1 && !raw;
  // FOLLOW: this op depends on its predecessor (single-item) and otherwise only
  // on ops that are the predecessor's ancestors in the same run or already done.
  bool follow = false;
  if (single && id > 0 && rt->prev_single) {
    const u64 p1 = id;  // encoded id + 1 of the predecessor (id - 1)
    if (dep[0] == p1 || dep[1] == p1) {
      const u64 other = dep[0] == p1 ? dep[1] : dep[0];
      follow = other == 0 || other == p1 || (other - 1 >= rt->prev_chain_start && other - 1 < id - 1) ||
               (other - 1 < rt->tail);
    }
  }
  e.dep0 = dep[0];
  e.dep1 = dep[1];
  e.prev_big = 0;
  if (items > 1) {
    e.prev_big = rt->last_big;
    rt->last_big = id + 1;
    rt->big_ids.push_back(id);
  }
  e.hdr = hdr_make(id, follow, items);
  bool fused = false;
  if (single && try_fuse(rt, id, rt->last_e, e)) {
    // the previous entry now computes both ops; this one only completes after it
    write_entry(rt, id - 1, rt->last_e);
    RingEntry nop;
    std::memset(&nop, 0, sizeof(nop));
    nop.opcode = GPUOS_OP_NOP;
    nop.rows = nop.cols = 1;
    nop.in_n0 = nop.in_n1 = 1;
    nop.dep0 = id;  // id - 1, encoded as id + 1 of it
    nop.hdr = hdr_make(id, follow, 1);
    e = nop;
    fused = true;
  }
  // write the 128-byte entry into the write-combined ring
  write_entry(rt, id, e);
  rt->last_e = e;
  rt->last_fusable = !fused && fusable(e, single);
  rt->prev_chain_start = follow ? rt->prev_chain_start : id;
  rt->prev_single = single;
  rt->next_id = id + 1;
  const u64 occ = rt->next_id - rt->tail;
  if (occ > rt->max_occ) rt->max_occ = occ;
  if (id_out) *id_out = id;
  return GPUOS_OK;
}

void free_all(gpuos* rt) {
  if (rt->hring) cudaFreeHost(rt->hring);
  if (rt->hctl) cudaFreeHost(rt->hctl);
  if (rt->hdone) cudaFreeHost(rt->hdone);
  if (rt->st) cudaFree(rt->st);
  if (rt->dring) cudaFree(rt->dring);
  if (rt->done) cudaFree(rt->done);
  if (rt->tiles_done) cudaFree(rt->tiles_done);
  if (rt->owner) cudaFree(rt->owner);
  if (rt->mbox) cudaFree(rt->mbox);
  if (rt->mctl) cudaFree(rt->mctl);
  if (rt->cstats) cudaFree(rt->cstats);
  if (rt->trace) cudaFree(rt->trace);
  if (rt->dma_ev) cudaEventDestroy(rt->dma_ev);
  if (rt->aux) cudaStreamDestroy(rt->aux);
}

}  // namespace

extern "C" {

gpuos_status gpuos_default_config(gpuos_config* cfg) {
  if (!cfg) return GPUOS_EINVAL;
  default_config(cfg);
  return GPUOS_OK;
}

gpuos_status gpuos_create(gpuos_stream_t stream, gpuos_t** out) { return gpuos_create_ex(stream, nullptr, out); }

gpuos_status gpuos_create_ex(gpuos_stream_t stream, const gpuos_config* cfg_in, gpuos_t** out) {
  if (!out) return GPUOS_EINVAL;
  *out = nullptr;
  gpuos_config cfg;
  if (cfg_in)
    cfg = *cfg_in;
  else
    default_config(&cfg);
  if (cfg.ring_capacity < 1024 || (cfg.ring_capacity & (cfg.ring_capacity - 1)) != 0) return GPUOS_EINVAL;
  if (cfg.elem_chunk < 1024 || cfg.elem_chunk % 1024 != 0 || cfg.row_chunk < 1) return GPUOS_EINVAL;
  if (cfg.timeout_ns < 1000000ull || cfg.idle_exit_ns < 1000000ull) return GPUOS_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPUOS_EDEVICE;
  int major = 0, sms = 0, canmap = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&canmap, cudaDevAttrCanMapHostMemory, dev) != cudaSuccess)
    return GPUOS_EDEVICE;
  if (major != 10 || !canmap) return GPUOS_EDEVICE;
  gpuos* rt = new (std::nothrow) gpuos();
  if (!rt) return GPUOS_ENOMEM;
  rt->dev = dev;
  rt->stream = static_cast<cudaStream_t>(stream);
  rt->cfg = cfg;
  rt->sms = (u32)sms;
  rt->grid = cfg.grid ? cfg.grid : (u32)sms;
  rt->cap = cfg.ring_capacity;
  rt->mask = rt->cap - 1;
  bool ok = cudaStreamCreateWithFlags(&rt->aux, cudaStreamNonBlocking) == cudaSuccess;
  ok = ok && cudaEventCreateWithFlags(&rt->dma_ev, cudaEventDisableTiming) == cudaSuccess;
  ok = ok && cudaHostAlloc((void**)&rt->hring, rt->cap * sizeof(RingEntry),
                           cudaHostAllocMapped | cudaHostAllocWriteCombined) == cudaSuccess;
  ok = ok && cudaHostAlloc((void**)&rt->hctl, sizeof(HostCtl), cudaHostAllocMapped) == cudaSuccess;
  ok = ok && cudaHostAlloc((void**)&rt->hdone, rt->cap * sizeof(u64), cudaHostAllocMapped) == cudaSuccess;
  if (ok) {
    std::memset(rt->hctl, 0, sizeof(HostCtl));
    std::memset(rt->hdone, 0, rt->cap * sizeof(u64));
    std::memset(rt->hring, 0, rt->cap * sizeof(RingEntry));
  }
  ok = ok && cudaHostGetDevicePointer((void**)&rt->hring_d, rt->hring, 0) == cudaSuccess;
  ok = ok && cudaHostGetDevicePointer((void**)&rt->hctl_d, rt->hctl, 0) == cudaSuccess;
  ok = ok && cudaHostGetDevicePointer((void**)&rt->hdone_d, rt->hdone, 0) == cudaSuccess;
  ok = ok && cudaMalloc((void**)&rt->st, sizeof(DevState)) == cudaSuccess;
  ok = ok && cudaMalloc((void**)&rt->dring, rt->cap * sizeof(RingEntry)) == cudaSuccess;
  ok = ok && cudaMalloc((void**)&rt->done, rt->cap * sizeof(u64)) == cudaSuccess;
  ok = ok && cudaMalloc((void**)&rt->tiles_done, rt->cap * sizeof(u32)) == cudaSuccess;
  ok = ok && cudaMalloc((void**)&rt->cstats, rt->grid * sizeof(CtaStats)) == cudaSuccess;
  ok = ok && cudaMalloc((void**)&rt->owner, rt->cap * sizeof(u64)) == cudaSuccess;
  ok = ok && cudaMalloc((void**)&rt->mbox, (size_t)rt->grid * MAILBOX * sizeof(u64)) == cudaSuccess;
  ok = ok && cudaMalloc((void**)&rt->mctl, rt->grid * sizeof(MailCtl)) == cudaSuccess;
  if (ok && (cfg.flags & GPUOS_CFG_TRACE))
    ok = cudaMalloc((void**)&rt->trace, rt->cap * sizeof(gpuos_trace_rec)) == cudaSuccess;
  ok = ok && cudaMemsetAsync(rt->st, 0, sizeof(DevState), rt->aux) == cudaSuccess;
  ok = ok && cudaMemsetAsync(rt->dring, 0, rt->cap * sizeof(RingEntry), rt->aux) == cudaSuccess;
  ok = ok && cudaMemsetAsync(rt->done, 0, rt->cap * sizeof(u64), rt->aux) == cudaSuccess;
  ok = ok && cudaMemsetAsync(rt->tiles_done, 0, rt->cap * sizeof(u32), rt->aux) == cudaSuccess;
  ok = ok && cudaMemsetAsync(rt->cstats, 0, rt->grid * sizeof(CtaStats), rt->aux) == cudaSuccess;
  ok = ok && cudaMemsetAsync(rt->owner, 0, rt->cap * sizeof(u64), rt->aux) == cudaSuccess;
  ok = ok && cudaStreamSynchronize(rt->aux) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_all(rt);
    delete rt;
    return GPUOS_ENOMEM;
  }
  if (!(cfg.flags & GPUOS_CFG_NO_AUTOSTART)) {
    const gpuos_status s = start_kernel(rt, 0);
    if (s != GPUOS_OK) {
      free_all(rt);
      delete rt;
      return s;
    }
  }
  *out = rt;
  return GPUOS_OK;
}

gpuos_status gpuos_start(gpuos_t* rt, uint32_t flags) {
  if (!rt || (flags & ~GPUOS_START_DRAIN)) return GPUOS_EINVAL;
  return start_kernel(rt, flags);
}

gpuos_status gpuos_stop(gpuos_t* rt, uint64_t timeout_ns) {
  if (!rt) return GPUOS_EINVAL;
  if (!rt->running) return rt->sticky;
  gpuos_status st = GPUOS_OK;
  if (rt->sticky == GPUOS_OK) {
    if (rt->run_flags & GPUOS_START_DRAIN)  // a drained session owes only the ops published at its start
      st = rt->run_head > rt->session_base ? wait_impl(rt, rt->run_head - 1, timeout_ns) : GPUOS_OK;
    else
      st = wait_impl(rt, GPUOS_ALL, timeout_ns);
  }
  if (!rt->running) return st == GPUOS_ESTOPPED ? GPUOS_OK : st;  // drained kernel already joined
  __atomic_store_n(&rt->hctl->stop, 1ull, __ATOMIC_RELEASE);
  const gpuos_status j = join_kernel(rt, (timeout_ns > rt->cfg.timeout_ns ? timeout_ns : rt->cfg.timeout_ns) * 2 +
                                             5000000000ull);
  if (j != GPUOS_OK) return j;
  if (st == GPUOS_OK && rt->sticky != GPUOS_OK) st = rt->sticky;
  return st;
}

gpuos_status gpuos_destroy(gpuos_t* rt) {
  if (!rt) return GPUOS_EINVAL;
  gpuos_status s = GPUOS_OK;
  if (rt->running) s = gpuos_stop(rt, rt->cfg.timeout_ns);
  if (rt->running) return GPUOS_EDEVICE;  // the kernel did not leave: its memory stays allocated
  free_all(rt);
  delete rt;
  return s == GPUOS_ESTOPPED ? GPUOS_OK : s;
}

gpuos_status gpuos_submit(gpuos_t* rt, const gpuos_desc* desc, uint64_t* id_out) {
  if (!rt) return GPUOS_EINVAL;
  return submit_one(rt, desc, GPUOS_NO_BASE, 0, reinterpret_cast<u64*>(id_out), false);
}

gpuos_status gpuos_submit_n(gpuos_t* rt, const gpuos_desc* descs, uint64_t n, uint64_t dep_base,
                            uint64_t* first_id_out) {
  if (!rt || (!descs && n)) return GPUOS_EINVAL;
  const u64 first = rt->next_id;
  if (first_id_out) *first_id_out = first;
  for (u64 i = 0; i < n; ++i) {
    const gpuos_status s = submit_one(rt, &descs[i], dep_base, first, nullptr, false);
    if (s != GPUOS_OK) return s;
  }
  return GPUOS_OK;
}

gpuos_status gpuos_flush(gpuos_t* rt) {
  if (!rt) return GPUOS_EINVAL;
  return flush_impl(rt);
}

gpuos_status gpuos_wait(gpuos_t* rt, uint64_t id, uint64_t timeout_ns) {
  if (!rt) return GPUOS_EINVAL;
  return wait_impl(rt, id, timeout_ns);
}

gpuos_status gpuos_query(gpuos_t* rt, uint64_t* completed) {
  if (!rt || !completed) return GPUOS_EINVAL;
  refresh_tail(rt);
  *completed = rt->tail;
  return rt->sticky;
}

gpuos_status gpuos_get_stats(gpuos_t* rt, gpuos_stats* o) {
  if (!rt || !o) return GPUOS_EINVAL;
  refresh_tail(rt);
  std::memset(o, 0, sizeof(*o));
  o->ops_submitted = rt->next_id;
  o->ops_completed = rt->tail;
  o->items_executed = rt->acc_items;
  o->ops_claimed = rt->acc_claimed;
  o->run_ops = rt->acc_run;
  o->idle_poll_cycles = rt->acc_idle;
  o->dep_wait_cycles = rt->acc_dep;
  o->fetch_descs = rt->acc_fetch;
  o->max_ring_occupancy = rt->max_occ;
  o->gpu_span_ns = rt->last_span;
  o->kernel_launches = rt->launches;
  o->num_ctas = rt->grid;
  o->last_error = (int32_t)rt->sticky;
  o->error_op = rt->err_op;
  return GPUOS_OK;
}

gpuos_status gpuos_trace_read(gpuos_t* rt, uint64_t first_id, uint64_t n, gpuos_trace_rec* out) {
  if (!rt || (!out && n)) return GPUOS_EINVAL;
  if (!rt->trace || rt->running || n > rt->cap) return GPUOS_EINVAL;
  std::vector<gpuos_trace_rec> all(rt->cap);
  if (cudaMemcpyAsync(all.data(), rt->trace, rt->cap * sizeof(gpuos_trace_rec), cudaMemcpyDeviceToHost, rt->aux) !=
          cudaSuccess ||
      cudaStreamSynchronize(rt->aux) != cudaSuccess)
    return GPUOS_EDEVICE;
  for (u64 i = 0; i < n; ++i) out[i] = all[(first_id + i) & rt->mask];
  return GPUOS_OK;
}

gpuos_status gpuos_launch_ops(const gpuos_desc* descs, uint64_t n, const gpuos_config* cfg_in,
                              gpuos_stream_t stream) {
  gpuos_config cfg;
  if (cfg_in)
    cfg = *cfg_in;
  else
    default_config(&cfg);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return GPUOS_EDEVICE;
  for (u64 i = 0; i < n; ++i) {
    const gpuos_status s = validate_desc(&descs[i], &cfg);
    if (s != GPUOS_OK || descs[i].opcode == GPUOS_OP_STALL) return GPUOS_EINVAL;
    RingEntry e;
    build_entry(&descs[i], &cfg, &e);
    if (launch_op(e, cfg.elem_chunk, cfg.row_chunk, (u32)sms, stream) != 0) return GPUOS_EDEVICE;
  }
  return GPUOS_OK;
}

struct gpuos_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

gpuos_status gpuos_graph_create(const gpuos_desc* descs, uint64_t n, uint64_t dep_base, const gpuos_config* cfg_in,
                                gpuos_stream_t stream, uint32_t mode, gpuos_graph_t** out, uint64_t* build_ns) {
  if (!out || (!descs && n) || mode > 1) return GPUOS_EINVAL;
  *out = nullptr;
  gpuos_config cfg;
  if (cfg_in)
    cfg = *cfg_in;
  else
    default_config(&cfg);
  const u64 t0 = now_ns();
  gpuos_graph* g = new (std::nothrow) gpuos_graph();
  if (!g) return GPUOS_ENOMEM;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (mode == 0) {
    if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
      delete g;
      return GPUOS_EDEVICE;
    }
    const gpuos_status ls = gpuos_launch_ops(descs, n, &cfg, stream);
    const cudaError_t ce = cudaStreamEndCapture(s, &g->graph);
    if (ls != GPUOS_OK || ce != cudaSuccess) {
      if (g->graph) cudaGraphDestroy(g->graph);
      delete g;
      cudaGetLastError();
      return ls != GPUOS_OK ? ls : GPUOS_EDEVICE;
    }
  } else {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaGraphCreate(&g->graph, 0) != cudaSuccess) {
      delete g;
      return GPUOS_EDEVICE;
    }
    std::vector<cudaGraphNode_t> nodes(n);
    for (u64 i = 0; i < n; ++i) {
      const gpuos_status vs = validate_desc(&descs[i], &cfg);
      if (vs != GPUOS_OK || descs[i].opcode == GPUOS_OP_STALL) {
        cudaGraphDestroy(g->graph);
        delete g;
        return GPUOS_EINVAL;
      }
      RingEntry e;
      build_entry(&descs[i], &cfg, &e);
      u32 gx, bx;
      op_launch_dims(e, cfg.elem_chunk, cfg.row_chunk, (u32)sms, &gx, &bx);
      u32 ec = cfg.elem_chunk, rc = cfg.row_chunk;
      void* args[3] = {&e, &ec, &rc};
      cudaKernelNodeParams kp;
      std::memset(&kp, 0, sizeof(kp));
      kp.func = op_kernel_fn();
      kp.gridDim = dim3(gx);
      kp.blockDim = dim3(bx);
      kp.sharedMemBytes = (unsigned)op_smem_bytes();
      kp.kernelParams = args;
      cudaGraphNode_t deps[2];
      size_t nd = 0;
      for (int k = 0; k < 2; ++k) {
        const u64 d = descs[i].dep[k];
        if (d == GPUOS_NO_DEP) continue;
        const u64 j = dep_base == GPUOS_NO_BASE ? d : d - dep_base;
        if (j >= i) {
          cudaGraphDestroy(g->graph);
          delete g;
          return GPUOS_EINVAL;
        }
        if (nd == 1 && deps[0] == nodes[j]) continue;
        deps[nd++] = nodes[j];
      }
      if (cudaGraphAddKernelNode(&nodes[i], g->graph, nd ? deps : nullptr, nd, &kp) != cudaSuccess) {
        cudaGraphDestroy(g->graph);
        delete g;
        cudaGetLastError();
        return GPUOS_EDEVICE;
      }
    }
  }
  if (cudaGraphInstantiate(&g->exec, g->graph, 0) != cudaSuccess) {
    cudaGraphDestroy(g->graph);
    delete g;
    cudaGetLastError();
    return GPUOS_EDEVICE;
  }
  if (build_ns) *build_ns = now_ns() - t0;
  *out = g;
  return GPUOS_OK;
}

gpuos_status gpuos_graph_launch(gpuos_graph_t* g, gpuos_stream_t stream) {
  if (!g) return GPUOS_EINVAL;
  return cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GPUOS_OK : GPUOS_EDEVICE;
}

gpuos_status gpuos_graph_destroy(gpuos_graph_t* g) {
  if (!g) return GPUOS_EINVAL;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
  return GPUOS_OK;
}

gpuos_status gpuos_validate(const gpuos_desc* desc) {
  gpuos_config cfg;
  default_config(&cfg);
  return validate_desc(desc, &cfg);
}

uint64_t gpuos_work_items(const gpuos_desc* desc, const gpuos_config* cfg_in) {
  gpuos_config cfg;
  if (cfg_in)
    cfg = *cfg_in;
  else
    default_config(&cfg);
  if (validate_desc(desc, &cfg) != GPUOS_OK) return 0;
  return op_items(desc->opcode, desc->rows, desc->cols, cfg.elem_chunk, cfg.row_chunk);
}

const char* gpuos_status_string(gpuos_status s) {
  switch (s) {
    case GPUOS_OK: return "ok";
    case GPUOS_EINVAL: return "invalid argument";
    case GPUOS_EAGAIN: return "ring full";
    case GPUOS_ETIMEDOUT: return "timed out";
    case GPUOS_EBADOP: return "unknown opcode on the device";
    case GPUOS_EDEVICE: return "CUDA or device error";
    case GPUOS_ESTOPPED: return "persistent kernel not running";
    case GPUOS_ENOMEM: return "out of memory";
  }
  return "unknown status";
}

gpuos_status gpuos_debug_submit_raw(gpuos_t* rt, const gpuos_desc* desc, uint64_t* id_out) {
  if (!rt) return GPUOS_EINVAL;
  return submit_one(rt, desc, GPUOS_NO_BASE, 0, reinterpret_cast<u64*>(id_out), true);
}

gpuos_status gpuos_debug_release_stall(gpuos_t* rt) {
  if (!rt) return GPUOS_EINVAL;
  __atomic_store_n(&rt->hctl->stall_gate, 1ull, __ATOMIC_RELEASE);
  return GPUOS_OK;
}

}  // extern "C"
