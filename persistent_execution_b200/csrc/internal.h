// internal.h -- layouts shared by the host runtime and the device code of the
// persistent op-queue runtime (not part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/gpuos.h"

#ifdef __CUDACC__
#define GPUOS_HD __host__ __device__ __forceinline__
#else
#define GPUOS_HD inline
#endif

namespace gpuos_impl {

typedef unsigned long long u64;
typedef unsigned int u32;

// Ring entry: the host-side form of one op after validation. 128 bytes. The
// host writes it into the pinned ring; a device fetcher copies it into the
// device ring and writes `hdr` last (release), so a reader that sees the tag
// of its id sees the whole entry.
struct __align__(16) RingEntry {
  u64 hdr;        //   0: (id + 1) << 24 | FOLLOW << 23 | items
  u64 dep0, dep1; //   8: id + 1 of a dependency, 0 = none
  u64 prev_big;   //  24: id + 1 of the previous multi-item op, 0 = none
  u64 in0, in1, in2, out;  // 32
  long long rows, cols;    // 64
  long long in_n0, in_n1;  // 80
  float s[4];              // 96
  int pos;                 // 112
  unsigned short opcode;   // 116
  unsigned char dtype, nmicro;  // 118
  unsigned char micro[8];  // 120
};
static_assert(sizeof(RingEntry) == 128, "ring entry is 128 bytes");

constexpr int HDR_TAG_SHIFT = 24;
constexpr u64 HDR_FOLLOW = 1ull << 23;
constexpr u64 HDR_ITEMS_MASK = (1ull << 23) - 1;
constexpr u64 MAX_ITEMS = HDR_ITEMS_MASK;

GPUOS_HD u64 hdr_make(u64 id, bool follow, u64 items) {
  return ((id + 1) << HDR_TAG_SHIFT) | (follow ? HDR_FOLLOW : 0ull) | items;
}
GPUOS_HD u64 hdr_tag(u64 h) { return h >> HDR_TAG_SHIFT; }  // id + 1
GPUOS_HD u64 hdr_items(u64 h) { return h & HDR_ITEMS_MASK; }
GPUOS_HD bool hdr_follow(u64 h) { return (h & HDR_FOLLOW) != 0; }

// Word of the currently open multi-item op: (id + 1) << 24 | items claimed.
constexpr u64 BIG_COUNT_MASK = (1ull << 24) - 1;
constexpr u64 BIG_EXHAUSTED = 1ull << 23;  // count that exceeds every op's items

// Internal micro-op (never accepted from callers): store the accumulator as an
// output at in1. The runtime fuses two consecutive dependent scalar elementwise
// ops A -> B into A's entry as progA, M_STORE1, progB (in1 = A's output, out =
// B's output) and turns B into a NOP that depends on A.
constexpr unsigned char M_STORE1 = 11;

GPUOS_HD bool op_is_row(int op) {
  return op == GPUOS_OP_ROWSUM || op == GPUOS_OP_ROWMAX || op == GPUOS_OP_SOFTMAX ||
         op == GPUOS_OP_RMSNORM || op == GPUOS_OP_LAYERNORM || op == GPUOS_OP_ROTARY;
}
GPUOS_HD bool op_is_ew(int op) {
  return op >= GPUOS_OP_ADD && op <= GPUOS_OP_EW_CHAIN;
}

GPUOS_HD long long rows_per_item(long long cols, u32 row_chunk) {
  // 32-bit division when cols fits (it always does below 2^32 columns)
  long long r = cols <= 0xffffffffll ? (long long)(row_chunk / (u32)cols) : 0;
  if (r < 1) r = 1;
  if (r > 1024) r = 1024;
  return r;
}

// Work items of one op: elementwise ops split their elements into chunks of
// elem_chunk; row ops split their rows into groups of rows_per_item.
GPUOS_HD u64 op_items(int op, long long rows, long long cols, u32 elem_chunk, u32 row_chunk) {
  if (op_is_ew(op)) {
    u64 n = (u64)rows * (u64)cols;
    return (n + elem_chunk - 1) / elem_chunk;
  }
  if (op_is_row(op)) {
    long long rpi = rows_per_item(cols, row_chunk);
    return (u64)((rows + rpi - 1) / rpi);
  }
  return 1;  // NOP, STALL
}

// A device counter on its own 128-byte line.
struct __align__(128) Line {
  u64 v;
  u64 pad[15];
};

// Device-resident scheduler state of the running session.
struct DevState {
  Line next_op;      // next op id to claim
  Line big;          // open multi-item op word
  Line fetch_next;   // next id to copy from the host ring
  Line head_mirror;  // host head as last read by the device
  Line poll_lock;    // one CTA at a time reads the host head
  Line poll_time;    // globaltimer of the last host poll
  Line stop;         // 1 = host asked to stop, 2 = idle exit
  Line abort_;       // 1 after the first device error
  Line ops_done;     // ops completed in this session
  Line err;          // first error: status | (id + 1) << 8
  Line activity;     // globaltimer of the last claim
  Line span_start;   // min item start
  Line span_end;     // max item end
  Line dma_mirror;   // dma_head as last read by the device
};

// Host control block in mapped pinned memory.
struct HostCtl {
  volatile u64 head;  // host -> device: ops [0, head) are published
  volatile u64 dma_head;  // host -> device: entries [0, dma_head) were copied into the device ring by the host
  u64 pad0[14];
  volatile u64 stop;        // host -> device
  volatile u64 stall_gate;  // host -> device: nonzero lets STALL ops finish
  u64 pad1[14];
  volatile u32 status;       // device -> host: first error (gpuos_status)
  volatile u32 exited_idle;  // device -> host: the kernel left after idling
  volatile u64 err_id;       // device -> host: id of the failing op
  u64 pad2[14];
};

struct CtaStats {
  u64 items, ops_claimed, run_ops, idle_cycles, dep_cycles, fetch_descs, pad[2];
};

// Warps of the compute group in a persistent CTA; the one-kernel-per-op
// baseline uses the same group size so both paths split rows identically.
constexpr int NCW = 16;

// Chain hand-off: a CTA that claims an op whose one unfinished dependency is
// running on another CTA posts the op to that CTA's mailbox, and the owner
// queues it right behind the dependency. owner[id & mask] = (id + 1) << 16 | cta
// of the CTA that emitted single-item op id; mailboxes hold id + 1, 0 = empty.
constexpr u32 MAILBOX = 16;
struct MailCtl {
  u64 tail;  // slots reserved by posting CTAs (CAS)
  u64 pad0[7];
  u64 head;  // slots taken by the owner
  u64 pad1[7];
};

constexpr u32 KF_DRAIN = 1u;
constexpr u32 KF_TRACE = 2u;
constexpr u32 KF_NO_BULK = 4u;  // op bodies use register paths only (no bulk-copy staging)

struct KParams {
  DevState* st;
  RingEntry* dring;
  u64* done;
  u32* tiles_done;
  const RingEntry* hring;  // device alias of the pinned host ring
  HostCtl* hctl;           // device alias of the host control block
  u64* hdone;              // device alias of the host completion array
  CtaStats* stats;
  gpuos_trace_rec* trace;
  u64* owner;     // [capacity], or null: no chain hand-off
  u64* mbox;      // [grid * MAILBOX]
  MailCtl* mctl;  // [grid]
  u64 mask;  // capacity - 1
  u64 base;  // first id of the session
  u64 fetched_upto;  // ids in [base, fetched_upto) are already in the device ring
  u64 timeout_ns;
  u64 idle_exit_ns;
  u32 elem_chunk, row_chunk, backoff_ns, flags, grid;
};

// Host-side launchers (persistent.cu, baseline.cu).
int launch_session(const KParams& p, u64 head, u64 big_init, void* stream);
int launch_op(const RingEntry& e, u32 elem_chunk, u32 row_chunk, u32 sms, void* stream);
void* op_kernel_fn();
size_t op_smem_bytes();
void op_launch_dims(const RingEntry& e, u32 elem_chunk, u32 row_chunk, u32 sms, u32* grid, u32* block);

}  // namespace gpuos_impl
