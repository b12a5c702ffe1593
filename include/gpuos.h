/*
 * gpuos.h -- C ABI of a persistent op-queue runtime for NVIDIA B200 (sm_100a).
 *
 * What it does. GPUOS (arXiv 2604.17861, "GPUOS: A GPU Operating System
 * Primitive for Transparent Operation Fusion", section "The Paper") runs one
 * long-lived GPU kernel that keeps taking tasks from a host-managed work queue,
 * so that a stream of small tensor ops costs no kernel launch per op. This
 * library is that primitive, re-designed for B200:
 *   - the host writes 128-byte op descriptors into a ring in mapped pinned
 *     memory and publishes a head counter (one doorbell per batch, in place of
 *     the per-launch ring write and doorbell of "Kernel Launch and
 *     Host-Device Interaction", section 5, "The launch path");
 *   - the descriptors reach a device ring by the copy engine (or, for small
 *     flushes to a running kernel, by the kernel itself);
 *   - one persistent kernel, one CTA per SM, claims ops and work items of
 *     large ops with atomics (the
 *     persistent worker and atomic task queues of the GPUOS abstract),
 *     waits for up to two dependencies per op through per-op completion words
 *     with acquire/release ordering, and runs each op body from an
 *     ahead-of-time opcode switch or a fused micro-op program held in
 *     registers ("Launch Overhead and Fusion", section "Fusion");
 *   - completion is published per op into mapped host memory, so waiting
 *     never needs a stream synchronisation ("Kernel Launch and Host-Device
 *     Interaction", section "Synchronization primitives").
 *
 * Conventions for every call:
 *   - All calls return a gpuos_status and never abort the process.
 *   - A device-side failure (dependency-wait timeout, unknown opcode, corrupted
 *     ring entry) is sticky: every later call on that runtime returns it;
 *     gpuos_destroy still releases everything.
 *   - Tensors are caller-owned device memory (for example from PyTorch's
 *     allocator). They must stay alive until the op that uses them completed
 *     (gpuos_wait on its id returned GPUOS_OK).
 *   - Streams are passed as gpuos_stream_t, the value of a cudaStream_t. The
 *     persistent kernel occupies its stream until it stops: use a dedicated
 *     non-blocking stream, never the legacy default stream.
 *   - A runtime is not thread-safe; use it from one host thread at a time.
 */
#ifndef GPUOS_H
#define GPUOS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gpuos gpuos_t;             /* opaque; owned by the library */
typedef struct gpuos_graph gpuos_graph_t; /* opaque; CUDA Graph baseline */
typedef void* gpuos_stream_t;             /* a cudaStream_t */

typedef enum {
  GPUOS_OK = 0,
  GPUOS_EINVAL = 1,    /* bad argument or descriptor; nothing was enqueued */
  GPUOS_EAGAIN = 2,    /* ring still full after the configured timeout */
  GPUOS_ETIMEDOUT = 3, /* a host wait, or a device dependency wait, ran out */
  GPUOS_EBADOP = 4,    /* the device met an opcode it does not know */
  GPUOS_EDEVICE = 5,   /* a CUDA call failed, no sm_100 device, or a corrupted ring entry */
  GPUOS_ESTOPPED = 6,  /* the persistent kernel is not running */
  GPUOS_ENOMEM = 7     /* an allocation failed */
} gpuos_status;

/* Element types. Every operand and the output of one op share the type;
 * arithmetic is fp32 (transcendentals of gelu and rotary in fp64), bf16
 * results are rounded to nearest-even once. */
enum { GPUOS_F32 = 0, GPUOS_BF16 = 1 };

/* Opcodes. n = rows * cols. Operand k is read at index (e mod in_n[k]) for
 * output element e when in_n[k] != n ("modulo broadcast"). */
enum {
  GPUOS_OP_NOP = 0,          /* completes without touching memory */
  GPUOS_OP_ADD = 1,          /* out = in0 + in1 */
  GPUOS_OP_MUL = 2,          /* out = in0 * in1 */
  GPUOS_OP_SCALE = 3,        /* out = s[0] * in0 */
  GPUOS_OP_GELU = 4,         /* out = 0.5 in0 (1 + erf(in0 / sqrt 2)) */
  GPUOS_OP_RELU_AFFINE = 5,  /* out = max(fmaf(s[0], in0, s[1]), +0); NaN passes */
  GPUOS_OP_SILU_MUL = 6,     /* out = in0 * sigmoid(in0) * in1 */
  GPUOS_OP_EW_CHAIN = 7,     /* fused micro-op program micro[0..nmicro) on in0 */
  GPUOS_OP_ROWSUM = 16,      /* in0 [rows, cols] -> out [rows] */
  GPUOS_OP_ROWMAX = 17,      /* in0 [rows, cols] -> out [rows]; NaN elements skipped */
  GPUOS_OP_SOFTMAX = 18,     /* per row of in0 [rows, cols] */
  GPUOS_OP_RMSNORM = 19,     /* x / sqrt(mean(x^2) + s[0]) * in1[col] */
  GPUOS_OP_LAYERNORM = 20,   /* (x - mean) / sqrt(var + s[0]) * in1[col] + in2[col], biased var */
  GPUOS_OP_ROTARY = 21,      /* in0 [heads, cols]: pairs (i, i + cols/2) turn by pos * s[0]^(-2i/cols) */
  GPUOS_OP_STALL = 250       /* test only: waits for gpuos_debug_release_stall or times out */
};

/* Micro-ops of GPUOS_OP_EW_CHAIN. The fp32 accumulator starts as in0[e] and is
 * rounded to fp32 after every micro-op; scalar micro-ops consume s[0..3] in
 * program order. */
enum {
  GPUOS_M_AFFINE = 1, /* acc = fmaf(s[k], acc, s[k+1]); k += 2 */
  GPUOS_M_SCALE = 2,  /* acc = acc * s[k]; k += 1 */
  GPUOS_M_ADDS = 3,   /* acc = acc + s[k]; k += 1 */
  GPUOS_M_RELU = 4,
  GPUOS_M_GELU = 5,
  GPUOS_M_SILU = 6,
  GPUOS_M_ADD1 = 7,   /* acc = acc + in1[e mod in_n[1]] */
  GPUOS_M_MUL1 = 8,
  GPUOS_M_ADD2 = 9,   /* acc = acc + in2[e] */
  GPUOS_M_MUL2 = 10
};

#define GPUOS_NO_DEP (~(uint64_t)0)
#define GPUOS_ALL (~(uint64_t)0)
#define GPUOS_NO_BASE (~(uint64_t)0)

/* One op. 128 bytes, plain old data; submit copies it. */
typedef struct gpuos_desc {
  uint16_t opcode;     /* GPUOS_OP_* */
  uint8_t dtype;       /* GPUOS_F32 or GPUOS_BF16 */
  uint8_t nmicro;      /* micro-ops used by GPUOS_OP_EW_CHAIN, 0..8 */
  uint32_t flags;      /* must be 0 */
  uint64_t dep[2];     /* ids of earlier ops this op waits for, or GPUOS_NO_DEP */
  const void* in[3];   /* device pointers of operands (unused ones may be NULL) */
  void* out;           /* device pointer of the output */
  int64_t rows, cols;  /* shape; elementwise ops may use rows = 1, cols = n */
  int64_t in_n[2];     /* element counts of in[0], in[1]; 0 means n */
  float s[4];          /* scalars, meaning per opcode */
  int32_t pos;         /* rotary position */
  uint8_t micro[8];    /* GPUOS_M_* program */
  uint32_t reserved0;  /* must be 0 */
  uint64_t reserved1;  /* must be 0 */
} gpuos_desc;

typedef struct gpuos_config {
  uint32_t ring_capacity;   /* descriptors in the ring; power of two >= 1024. Default 131072 */
  uint32_t grid;            /* persistent CTAs; 0 = one per SM */
  uint64_t timeout_ns;      /* budget of every device wait on another op. Default 2 s */
  uint64_t submit_timeout_ns; /* how long gpuos_submit waits for ring space. Default 2 s */
  uint64_t idle_exit_ns;    /* kernel exits after this long with nothing to do (flush relaunches it). Default 20 s */
  uint32_t elem_chunk;      /* elements per work item of elementwise ops; multiple of 1024. Default 262144 */
  uint32_t row_chunk;       /* target elements per work item of row ops; rows per item = clamp(row_chunk/cols, 1, 1024). Default 524288 */
  uint32_t backoff_ns;      /* longest sleep of an idle poll. Default 1000 */
  uint32_t flags;           /* GPUOS_CFG_* */
} gpuos_config;

#define GPUOS_CFG_NO_AUTOSTART 1u /* gpuos_create_ex does not launch the kernel */
#define GPUOS_CFG_TRACE 2u        /* record a per-op event log (gpuos_trace_read) */
#define GPUOS_CFG_NO_BULK 4u      /* op bodies read operands with plain loads only, no bulk-copy staging */
#define GPUOS_CFG_NO_HANDOFF 8u   /* no chain hand-off: a claimed op always waits for its dependencies where it was claimed */
#define GPUOS_CFG_NO_FUSION 16u   /* no fused pairs: every submitted op runs as its own entry */

#define GPUOS_START_DRAIN 1u      /* the kernel exits once every op published before gpuos_start completed */

typedef struct gpuos_stats {
  uint64_t ops_submitted;     /* since create */
  uint64_t ops_completed;     /* contiguous completed prefix length since create */
  uint64_t items_executed;    /* work items run by the persistent kernel, all sessions */
  uint64_t ops_claimed;       /* ops claimed through the shared claim counter */
  uint64_t run_ops;           /* ops taken by chain affinity (claimed as a run by the CTA that ran the predecessor) */
  uint64_t idle_poll_cycles;  /* SM cycles spent polling with nothing to do, summed over CTAs */
  uint64_t dep_wait_cycles;   /* SM cycles spent waiting for another CTA's op, summed over CTAs */
  uint64_t fetch_descs;       /* descriptors the kernel copied from the host ring itself */
  uint64_t max_ring_occupancy;
  uint64_t gpu_span_ns;       /* last session: first item start to last item end (device globaltimer) */
  uint64_t kernel_launches;   /* kernels launched by this runtime */
  uint32_t num_ctas;
  int32_t last_error;         /* gpuos_status of the sticky error, 0 if none */
  uint64_t error_op;          /* id of the op that raised it */
} gpuos_stats;

typedef struct gpuos_trace_rec {
  uint64_t id;      /* op id + 1; 0 = no record */
  uint64_t t_start; /* earliest item start, device ns */
  uint64_t t_end;   /* latest item end, device ns */
  uint32_t cta;     /* CTA that ran the last item */
  uint32_t smid;
  uint32_t items;   /* items run */
  uint32_t claim;   /* how the op reached its CTA: 0 shared claim, 1 chain run, 2 large-op item, 3 chain hand-off */
} gpuos_trace_rec;

/* ---------------------------------------------------------------- lifecycle */

/* Fills *cfg with the defaults above. Needs no GPU. */
gpuos_status gpuos_default_config(gpuos_config* cfg);

/* Allocates the ring (pinned, mapped), the device tables, and launches the
 * persistent kernel on `stream` (one CTA per SM). The stream must belong to the
 * current device, which must be compute capability 10.x. */
gpuos_status gpuos_create(gpuos_stream_t stream, gpuos_t** out);
gpuos_status gpuos_create_ex(gpuos_stream_t stream, const gpuos_config* cfg, gpuos_t** out);

/* Launches the persistent kernel again after gpuos_stop (or after create with
 * GPUOS_CFG_NO_AUTOSTART). With GPUOS_START_DRAIN it runs the ops published by
 * gpuos_flush before this call and exits by itself; ops submitted later wait
 * for the next start. Before a drained launch the session's descriptors are
 * copied into device memory (ordered before the kernel on `stream`). Returns
 * GPUOS_EINVAL if it is already running. */
gpuos_status gpuos_start(gpuos_t* rt, uint32_t flags);

/* Waits (up to timeout_ns) for the session's work -- every submitted op, or
 * for a GPUOS_START_DRAIN session the ops published before its start -- then
 * asks the kernel to exit and waits for it. Ops submitted but not yet run
 * stay in the ring for the next gpuos_start. The runtime keeps its memory. */
gpuos_status gpuos_stop(gpuos_t* rt, uint64_t timeout_ns);

/* gpuos_stop, then frees everything. Safe on a runtime with a sticky error. */
gpuos_status gpuos_destroy(gpuos_t* rt);

/* ---------------------------------------------------------------- queue */

/* Validates and copies one descriptor into the ring; *id_out (may be NULL)
 * receives its id. Ids are dense, start at 0 and grow by one per submit. Each
 * dependency must be an earlier id, else GPUOS_EINVAL. When the ring is full,
 * submit flushes and waits up to timeout_ns for space, then GPUOS_EAGAIN
 * (immediately when the kernel is not running). Nothing becomes visible to
 * the device before gpuos_flush. */
gpuos_status gpuos_submit(gpuos_t* rt, const gpuos_desc* desc, uint64_t* id_out);

/* Submits descs[0..n) in order. When dep_base != GPUOS_NO_BASE, dependencies
 * are numbers in the caller's own numbering of ops, in which descs[0] has
 * number dep_base: dependency d (other than GPUOS_NO_DEP) names the op with
 * id first_id + d - dep_base, which may lie in an earlier call. This is the
 * form a prebuilt stream can be resubmitted in, in one call or in batches.
 * Stops at the first failing descriptor; *first_id_out receives descs[0]'s id. */
gpuos_status gpuos_submit_n(gpuos_t* rt, const gpuos_desc* descs, uint64_t n, uint64_t dep_base,
                            uint64_t* first_id_out);

/* Publishes every submitted op to the device: one release fence and one store
 * of the head counter into mapped memory. Relaunches a kernel that left after
 * idling. The new descriptors reach device memory by the copy engine (on an
 * internal stream) when no kernel or a drained one is running, and, for a live
 * kernel, when at least 128 ops are new: this call then waits for that copy
 * before moving the head, so the kernel never reads descriptors over PCIe
 * while ops run. Smaller flushes to a live kernel are fetched by the kernel. */
gpuos_status gpuos_flush(gpuos_t* rt);

/* Waits until op `id` (GPUOS_ALL: every submitted op) and every earlier op
 * completed; their outputs are then visible to later work on any stream.
 * Flushes first when needed. Polls mapped memory; makes no CUDA call. */
gpuos_status gpuos_wait(gpuos_t* rt, uint64_t id, uint64_t timeout_ns);

/* Length of the completed prefix of ids, without waiting. */
gpuos_status gpuos_query(gpuos_t* rt, uint64_t* completed);

/* Counters; device counters are read while the kernel is stopped or running. */
gpuos_status gpuos_get_stats(gpuos_t* rt, gpuos_stats* out);

/* Copies event-log records of ops [first_id, first_id + n) (GPUOS_CFG_TRACE;
 * the log keeps the last ring_capacity ops). The kernel must be stopped. */
gpuos_status gpuos_trace_read(gpuos_t* rt, uint64_t first_id, uint64_t n, gpuos_trace_rec* out);

/* ---------------------------------------------------------------- baselines */

/* The same op bodies, one kernel launch per op, in array order on `stream`
 * (the one-launch-per-op path of "Kernel Launch and Host-Device Interaction",
 * section 5). Dependencies are implied by stream order. Asynchronous. */
gpuos_status gpuos_launch_ops(const gpuos_desc* descs, uint64_t n, const gpuos_config* cfg,
                              gpuos_stream_t stream);

/* Records the launches of gpuos_launch_ops into a CUDA Graph ("Launch Overhead
 * and Fusion", section "Graph capture"). mode 0: stream capture of the
 * launches in order (a chain of kernel nodes); mode 1: one kernel node per op
 * with an edge per dependency, dependency d naming descs[d - dep_base], so
 * independent ops may overlap. *build_ns receives capture + instantiation time. */
gpuos_status gpuos_graph_create(const gpuos_desc* descs, uint64_t n, uint64_t dep_base,
                                const gpuos_config* cfg, gpuos_stream_t stream, uint32_t mode,
                                gpuos_graph_t** out, uint64_t* build_ns);
gpuos_status gpuos_graph_launch(gpuos_graph_t* g, gpuos_stream_t stream);
gpuos_status gpuos_graph_destroy(gpuos_graph_t* g);

/* ---------------------------------------------------------------- allocation-free variant */

/* The pages have no counterpart of this call; it exists for callers that must
 * not allocate. cudaMalloc, cudaHostAlloc and cudaFree can stall the whole
 * device for milliseconds and fail when another allocator (PyTorch's caching
 * allocator, for example) already holds the memory, so a latency-critical
 * caller, or one whose device memory belongs to someone else, cannot use
 * gpuos_create. gpuos_run_static runs descs[0..n) as one drained session of
 * the persistent kernel without allocating anything: the ring, completion
 * words and scheduler state live in a fixed array of about 620 KB inside the
 * library (every GPU that loads the library holds it until the process exits).
 *   - n <= 4096 and no GPUOS_OP_STALL ops, else GPUOS_EINVAL; at most 256 CTAs.
 *   - Dependencies are indices into descs (an index below the op's own).
 *   - Tensors are caller-owned device memory, as for gpuos_submit.
 *   - Synchronous: returns once every op completed (or a device error, which
 *     is returned, not kept). Uses `stream` for its copies and launches.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - Every call uses the same array and leaves it as the last call left it
 *     (each call clears what must start at zero). Calls that overlap on the
 *     GPU -- from two host threads, or on two streams -- race and corrupt
 *     each other's state. */
gpuos_status gpuos_run_static(const gpuos_desc* descs, uint64_t n, const gpuos_config* cfg,
                              gpuos_stream_t stream);

/* ---------------------------------------------------------------- host-only helpers */

/* Checks a descriptor as gpuos_submit does, without a runtime or GPU. */
gpuos_status gpuos_validate(const gpuos_desc* desc);

/* Work items the op is split into under cfg (NULL = defaults). 0 if invalid. */
uint64_t gpuos_work_items(const gpuos_desc* desc, const gpuos_config* cfg);

const char* gpuos_status_string(gpuos_status s);

/* ---------------------------------------------------------------- test hooks */

/* Writes a raw 128-byte ring entry for the next id without validation (its
 * header is filled in). Used to show that the device rejects a bad opcode with
 * GPUOS_EBADOP instead of faulting. */
gpuos_status gpuos_debug_submit_raw(gpuos_t* rt, const gpuos_desc* desc, uint64_t* id_out);

/* Lets every GPUOS_OP_STALL op that is waiting, or will wait, complete. */
gpuos_status gpuos_debug_release_stall(gpuos_t* rt);

#ifdef __cplusplus
}
#endif
#endif
