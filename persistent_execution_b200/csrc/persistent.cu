// persistent.cu -- the persistent op-queue kernel (one CTA per SM) and its reset kernel.
//
// GPUOS ("GPUOS: A GPU Operating System Primitive for Transparent Operation
// Fusion", section "The Paper") keeps one kernel alive that takes tasks from a
// host-managed queue through atomic task queues. On B200 each CTA is split
// into three warp roles that overlap with one another:
//
//   warp 0, control:   copies descriptors from the pinned host ring into device
//                      memory, claims ops (shared claim counter) and work items
//                      of large ops, waits for dependencies, and hands items to
//                      the compute warps through a shared-memory FIFO;
//   warp 1, publisher: after the compute warps finish an item, fences and
//                      publishes the op's completion word (device scope, for
//                      dependants) and its completion entry in mapped host
//                      memory (system scope, for gpuos_wait);
//   warps 2..17:       compute; run op bodies (ops.cuh).
//
// Chain affinity: the CTA that runs op c claims the next ops as one run when
// each depends only on its predecessor (FOLLOW flag, set by the host), so a
// dependent chain stays on one SM with no cross-SM hand-off per op.
//
// Large ops: an op split into several items is "opened" in a single word
// (id, items claimed) that every CTA can join with one atomicAdd; large ops open
// in submission order, which keeps the claim order deadlock-free (the same
// guarantee LithOS states for its atomizer: non-overlapping block ranges, each
// block run exactly once -- LithOS summary, section 5.4, Algorithm 1).
//
// Every wait on another CTA is bounded by timeout_ns and reports
// GPUOS_ETIMEDOUT through the status word instead of hanging; idle waits end
// on stop, drain or idle exit.
#include <cuda_runtime.h>

#include "internal.h"
#include "ops.cuh"
#include "ptx.cuh"

namespace gpuos_impl {

constexpr int NTHREADS = (NCW + 2) * 32;
constexpr int FIFO = 8;
// Items a CTA may have emitted but not finished before it claims another op
// or joins a large op: a shallow window keeps ready ops from queueing behind
// unrelated ones and keeps a large op's items from being hoarded long before
// they run, while a claim (several round trips) still overlaps the items
// ahead of it. Runs of FOLLOW ops use the whole FIFO. (2 -> 4: the 20,000-op
// DAG 1.13 -> 1.03 ms; chains and the serving stream unchanged.)
constexpr unsigned LOOKAHEAD = 4;
constexpr unsigned LOOKAHEAD_BIG = 2;  // joining a large op (large-op stress: 16.5 ms at 4, 15.5 at 2)
constexpr unsigned FULLMASK = 0xffffffffu;

enum : u32 { SLOT_WORK = 0, SLOT_EXIT = 1 };
enum : u32 { CLAIM_SHARED = 0, CLAIM_RUN = 1, CLAIM_BIG = 2, CLAIM_MAIL = 3 };

struct __align__(16) Slot {
  RingEntry e;
  u64 id;
  u32 item, nitems;
  u32 kind, claim;
  u64 t_start, t_end;
  u64 pad;
};

struct Smem {
  Slot slot[FIFO];
  RingEntry stage[32];  // descriptors of the run claimed by try_extend
  u64 full_bar[FIFO];
  u64 done_bar[FIFO];
  u64 free_bar[FIFO];
  float4 part[NCW];
  u64 recent[8];
  u64 deferred[32];         // mailbox ops waiting for the op this CTA holds (ids)
  RotCache rot;             // rotary angles of the last rotary op
  volatile unsigned ncomp;  // items the compute warps finished
};
constexpr u32 DEFER = 32;

__device__ __forceinline__ u64 bcast(u64 v) { return __shfl_sync(FULLMASK, v, 0); }
__device__ __forceinline__ u32 bcast32(u32 v) { return __shfl_sync(FULLMASK, v, 0); }

// ------------------------------------------------------------------ control warp
struct Control {
  const KParams& p;
  Smem* S;
  int lane;
  u64 k = 0;                      // items emitted
  u64 run_next = 0, run_end = 0;  // claimed run of FOLLOW ops
  u64 run_first = 0;              // op of stage[0]
  u64 pending = 0;                // id + 1 of a large op waiting to open
  u64 pend_word = 0, pend_t = 0;  // progress watchdog of the pending open
  u64 dep_ok = 0;                 // id + 1 of the large op whose dependencies were seen
  bool has_run = false;
  u64 lo = 0, hi = 0;             // contiguous single-item ops emitted by this CTA
  u32 nrecent = 0, rix = 0;
  u32 backoff = 0;
  u32 iters = 0;
  u64 claimed = 0, runops = 0, idle_cyc = 0, dep_cyc = 0, fetched = 0;
  u64 mb_head = 0;                // mailbox slots this CTA has taken
  u64 held = 0;                   // id + 1 of the single op claimed here and not yet emitted
  bool contended = false;         // this CTA lost a CAS claim race in this session (lane 0)
  u32 ndef = 0;                   // entries of S->deferred
  const bool drain;

  __device__ Control(const KParams& pp, Smem* s, int l) : p(pp), S(s), lane(l), drain((pp.flags & KF_DRAIN) != 0) {}

  __device__ __forceinline__ RingEntry* ent(u64 id) const { return &p.dring[id & p.mask]; }
  __device__ __forceinline__ u64 hdr_of(u64 id) const { return ld_acquire_gpu(&ent(id)->hdr); }

  __device__ __forceinline__ bool aborted() const { return ld_relaxed_gpu(&p.st->abort_.v) != 0; }

  __device__ __forceinline__ bool is_local(u64 d) const {
    if (has_run && d >= lo && d <= hi) return true;
    const bool hit = lane < 8 && (u32)lane < nrecent && S->recent[lane] == d;
    return __any_sync(FULLMASK, hit);
  }

  __device__ __forceinline__ void note_single(u64 c) {
    if (has_run && c == hi + 1) {
      hi = c;
    } else {
      has_run = true;
      lo = hi = c;
    }
    if (lane == 0) S->recent[rix & 7] = c;
    __syncwarp();
    ++rix;
    nrecent = nrecent + 1 > 8 ? 8 : nrecent + 1;
  }

  // Mailbox slot this CTA reads next.
  __device__ __forceinline__ u64* mail_slot() const { return &p.mbox[(u64)blockIdx.x * MAILBOX + (mb_head % MAILBOX)]; }
  __device__ __forceinline__ bool mail_ready() const { return p.mbox && ld_acquire_gpu(mail_slot()) != 0; }

  // Lane 0: polls the completion words of d0, d1 (id + 1, 0 = none) and the
  // mailbox. 1 = both done, 2 = an op arrived in the mailbox, 0 = abort or
  // timeout (timed from t0).
  __device__ __forceinline__ u32 spin_deps(u64 id, u64 d0, u64 d1, u64 t0, bool mail = true) {
    const u64* w0 = d0 ? &p.done[(d0 - 1) & p.mask] : nullptr;
    const u64* w1 = d1 ? &p.done[(d1 - 1) & p.mask] : nullptr;
    const u64 c0 = clock64();
    u32 r = 0;
    for (u32 spins = 0;; ++spins) {
      const bool ok0 = !w0 || ld_acquire_gpu(w0) >= d0;
      const bool ok1 = !w1 || ld_acquire_gpu(w1) >= d1;
      if (ok0 && ok1) {
        r = 1;
        break;
      }
      if (mail && mail_ready()) {
        r = 2;
        break;
      }
      if ((spins & 63) == 63) {
        if (aborted()) break;
        if (globaltimer() - t0 > p.timeout_ns) {
          raise_error(p.st, p.hctl, GPUOS_ETIMEDOUT, id);
          break;
        }
      }
      if (spins > 64) __nanosleep(spins > 4096 ? 256 : 32);
    }
    dep_cyc += clock64() - c0;
    return r;
  }

  // Waits until both dependencies (id + 1, 0 = none) of op id completed; ops
  // that arrive in the mailbox meanwhile are queued first (one of them may be
  // what id waits for). False on abort or timeout.
  __device__ __forceinline__ bool wait_deps(u64 id, u64 d0, u64 d1) {
    if (d0 != 0 && is_local(d0 - 1)) d0 = 0;
    if (d1 != 0 && is_local(d1 - 1)) d1 = 0;
    if ((d0 | d1) == 0) return true;
    const u64 t0 = lane == 0 ? globaltimer() : 0ull;
    bool mail = true;
    for (;;) {
      u32 r = 0;
      if (lane == 0) r = spin_deps(id, d0, d1, t0, mail);
      r = bcast32(r);
      if (r == 1) return true;
      if (r == 0) return false;
      const int m = serve_mail(false);
      if (m < 0) return false;
      if (m == 0) mail = false;  // nothing could be taken (deferred list full): wait without the mailbox
    }
  }

  __device__ __forceinline__ void set_owner(u64 c) {
    if (p.owner && lane == 0) st_relaxed_gpu(&p.owner[c & p.mask], ((c + 1) << 16) | (u64)blockIdx.x);
  }

  // Queues a mailbox op: emitted, owned here from now on.
  __device__ __forceinline__ bool emit_mail(u64 c) {
    if (!emit(c, 0, 1, CLAIM_MAIL)) return false;
    note_single(c);
    set_owner(c);
    return true;
  }

  // Takes the next op from this CTA's mailbox, if any. The poster saw every
  // dependency but one complete, and that one owned here: emitted (the op
  // then runs after it in FIFO order) or held (the op is deferred until the
  // held op is emitted). -1 error, 0 empty, 1 taken.
  // extend: also claim the FOLLOW ops after it as a run (only where no run or
  // claimed op is in progress).
  __device__ __forceinline__ int serve_mail(bool extend) {
    if (!p.mbox || ndef >= DEFER) return 0;
    u64 v = 0, d0 = 0, d1 = 0;
    if (lane == 0) {
      u64* slot = mail_slot();
      v = ld_acquire_gpu(slot);
      if (v != 0) {
        st_relaxed_gpu(slot, 0ull);
        st_release_gpu(&p.mctl[blockIdx.x].head, mb_head + 1);  // the slot is free again
        d0 = ent(v - 1)->dep0;
        d1 = ent(v - 1)->dep1;
      }
    }
    v = bcast(v);
    if (v == 0) return 0;
    ++mb_head;
    const u64 c = v - 1;
    d0 = bcast(d0);
    d1 = bcast(d1);
    if (held != 0 && (waits_held(d0) || waits_held(d1))) {
      if (lane == 0) S->deferred[ndef] = c;
      __syncwarp();
      ++ndef;
      return 1;
    }
    // the dependency is local or done; anything else is waited for here
    if (d0 != 0 && is_local(d0 - 1)) d0 = 0;
    if (d1 != 0 && is_local(d1 - 1)) d1 = 0;
    if ((d0 | d1) != 0) {
      u32 r = 0;
      if (lane == 0) r = spin_deps(c, d0, d1, globaltimer(), false);
      if (bcast32(r) != 1) return -1;
    }
    if (!emit_mail(c)) return -1;
    if (extend && run_next >= run_end) try_extend(c);
    return 1;
  }

  // True if d (id + 1) is the held op or a mailbox op deferred behind it.
  __device__ __forceinline__ bool waits_held(u64 d) {
    if (d == 0) return false;
    if (d == held) return true;
    const bool hit = (u32)lane < ndef && S->deferred[lane] + 1 == d;
    return __any_sync(FULLMASK, hit);
  }

  // After the held op is emitted: the mailbox ops that waited for it.
  __device__ __forceinline__ bool release_held() {
    held = 0;
    for (u32 i = 0; i < ndef; ++i) {
      u64 c = 0;
      if (lane == 0) c = S->deferred[i];
      if (!emit_mail(bcast(c))) return false;
    }
    ndef = 0;
    return true;
  }

  // Posts single-item op c, whose dependencies are d0, d1 (id + 1, 0 = none),
  // to the CTA that emitted its one unfinished dependency. True if posted;
  // false leaves c to the caller (nothing to wait for, two unfinished
  // dependencies, an unknown or local owner, or a full mailbox).
  // HO_POSTED: posted. HO_READY: every dependency already completed (read with
  // acquire ordering, so the caller needs no wait). HO_NONE: the caller waits.
  enum { HO_NONE = 0, HO_POSTED = 1, HO_READY = 2 };
  __device__ __forceinline__ int try_handoff(u64 c, u64 d0, u64 d1) {
    if ((d0 | d1) == 0) return HO_READY;
    if (!p.mbox) return HO_NONE;
    if ((d0 != 0 && is_local(d0 - 1)) || (d1 != 0 && is_local(d1 - 1))) return HO_NONE;
    u32 ok = HO_NONE;
    if (lane == 0) {
      const bool u0 = d0 != 0 && ld_acquire_gpu(&p.done[(d0 - 1) & p.mask]) < d0;
      const bool u1 = d1 != 0 && ld_acquire_gpu(&p.done[(d1 - 1) & p.mask]) < d1;
      if (!u0 && !u1) ok = HO_READY;
      if (u0 != u1) {
        const u64 a = u0 ? d0 : d1;
        const u64 o = ld_relaxed_gpu(&p.owner[(a - 1) & p.mask]);
        const u32 cta = (u32)(o & 0xffffu);
        if ((o >> 16) == a && cta != blockIdx.x && cta < p.grid) {
          MailCtl* m = &p.mctl[cta];
          const u64 t = ld_relaxed_gpu(&m->tail);
          const u64 h = ld_acquire_gpu(&m->head);
          if (t - h < MAILBOX && atomicCAS(&m->tail, t, t + 1) == t) {
            st_release_gpu(&p.mbox[(u64)cta * MAILBOX + (t % MAILBOX)], c + 1);
            // c is owned there from now on: its own dependants follow it
            st_relaxed_gpu(&p.owner[c & p.mask], ((c + 1) << 16) | (u64)cta);
            ok = HO_POSTED;
          }
        }
      }
    }
    return (int)bcast32(ok);
  }

  // Waits until this CTA has fewer than `lim` items emitted but not finished.
  // Mailbox ops that arrive meanwhile are queued at once. False on error.
  __device__ __forceinline__ bool throttle(unsigned lim) {
    bool mail = p.mbox != nullptr;
    for (;;) {
      u32 r = 0;
      if (lane == 0) {
        for (u32 spins = 0; (unsigned)k - S->ncomp >= lim; ++spins) {
          if (mail && (spins & 15) == 15 && mail_ready()) {  // a global load: not on every spin
            r = 1;
            break;
          }
          __nanosleep(20);
        }
      }
      if (bcast32(r) == 0) return true;
      const int m = serve_mail(true);
      if (m < 0) return false;
      if (m == 0) mail = false;
    }
  }

  // Copies one entry into the next FIFO slot and signals the compute warps.
  // The caller has read the entry's tag with acquire ordering (lane 0, or the
  // staging lane); the warp barrier below orders every copying lane after it.
  __device__ __forceinline__ bool emit(u64 id, u32 item, u32 nitems, u32 claim, const RingEntry* staged = nullptr,
                                       bool have_reg = false, uint4 reg = uint4{0, 0, 0, 0}) {
    const u32 slot = (u32)(k % FIFO);
    const u32 par = (u32)((k / FIFO) & 1) ^ 1u;
    u32 ok = 1;
    if (lane == 0) {
      const u64 t0 = globaltimer();
      for (u32 spins = 0; !mbar_try_wait(&S->free_bar[slot], par); ++spins) {
        if ((spins & 255) == 255 && globaltimer() - t0 > 2 * p.timeout_ns + 1000000000ull) {
          raise_error(p.st, p.hctl, GPUOS_ETIMEDOUT, id);
          ok = 0;
          break;
        }
      }
    }
    if (bcast32(ok) == 0) return false;
    Slot& s = S->slot[slot];
    __syncwarp();
    if (lane < 8) {
      if (have_reg)
        reinterpret_cast<uint4*>(&s.e)[lane] = reg;
      else if (staged)
        reinterpret_cast<uint4*>(&s.e)[lane] = reinterpret_cast<const uint4*>(staged)[lane];
      else
        reinterpret_cast<uint4*>(&s.e)[lane] = __ldcg(reinterpret_cast<const uint4*>(ent(id)) + lane);
    }
    if (lane == 0) {
      s.id = id;
      s.item = item;
      s.nitems = nitems;
      s.kind = SLOT_WORK;
      s.claim = claim;
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&S->full_bar[slot]);
      st_relaxed_gpu(&p.st->activity.v, globaltimer());
    }
    ++k;
    return true;
  }

  __device__ __forceinline__ void emit_exit() {
    const u32 slot = (u32)(k % FIFO);
    const u32 par = (u32)((k / FIFO) & 1) ^ 1u;
    if (lane == 0) {
      const u64 t0 = globaltimer();
      for (u32 spins = 0; !mbar_try_wait(&S->free_bar[slot], par); ++spins) {
        if ((spins & 255) == 255 && globaltimer() - t0 > 4 * p.timeout_ns + 2000000000ull) break;
      }
      S->slot[slot].kind = SLOT_EXIT;
      S->slot[slot].id = ~0ull;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S->full_bar[slot]);
    ++k;
  }

  // Copies up to 32 published descriptors from the host ring. True if fetch
  // work was available (done by this CTA or another one).
  __device__ __forceinline__ bool help_fetch() {
    u64 fn = 0, e = 0;
    u32 got = 0;
    if (lane == 0) {
      fn = ld_relaxed_gpu(&p.st->fetch_next.v);
      const u64 hm = ld_acquire_gpu(&p.st->head_mirror.v);
      if (drain && fn < hm) {
        // drained session: the head is fixed, so every CTA takes its own
        // batch at once; a batch that starts at or past the head is empty
        fn = atomicAdd(&p.st->fetch_next.v, 32ull);
        e = fn + 32 < hm ? fn + 32 : hm;
        got = fn < hm;
        if (!got) e = fn;
      } else if (fn < hm) {
        const u64 dm = ld_acquire_gpu(&p.st->dma_mirror.v);
        if (fn < dm) {
          // the host already copied these entries into the device ring: skip them
          atomicCAS(&p.st->fetch_next.v, fn, dm);
          e = fn + 1;  // progress, nothing to copy
        } else {
          e = fn + 32 < hm ? fn + 32 : hm;
          got = atomicCAS(&p.st->fetch_next.v, fn, e) == fn;
          if (!got) e = fn + 1;  // someone else took it: still progress
        }
      }
    }
    fn = bcast(fn);
    e = bcast(e);
    got = bcast32(got);
    if (!got) return e > fn;
    const u64 id = fn + (u64)lane;
    bool bad = false;
    if (id < e) {
      const uint4* src = reinterpret_cast<const uint4*>(&p.hring[id & p.mask]);
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = ld_volatile_v4(src + j);
      const u64 h = (u64)v[0].x | ((u64)v[0].y << 32);
      if (hdr_tag(h) != id + 1) {
        bad = true;
      } else {
        RingEntry* dst = ent(id);
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int j = 1; j < 8; ++j) d4[j] = v[j];
        dst->dep0 = (u64)v[0].z | ((u64)v[0].w << 32);
        st_release_gpu(&dst->hdr, h);
      }
    }
    const unsigned badm = __ballot_sync(FULLMASK, bad);
    if (badm && lane == 0) raise_error(p.st, p.hctl, GPUOS_EDEVICE, fn + (u64)(__ffs(badm) - 1));
    fetched += e - fn;
    return true;
  }

  // One CTA at a time reads the host head and stop word over PCIe and mirrors them.
  __device__ __forceinline__ void poll_host(u64 now) {
    if (drain || lane != 0) return;
    if (now - ld_relaxed_gpu(&p.st->poll_time.v) < 1000) return;
    if (atomicCAS(&p.st->poll_lock.v, 0ull, 1ull) != 0) return;
    const u64 h = ld_acquire_sys(&p.hctl->head);
    const u64 dh = ld_relaxed_sys(&p.hctl->dma_head);  // written before head
    const u64 sp = ld_relaxed_sys(&p.hctl->stop);
    if (dh > ld_relaxed_gpu(&p.st->dma_mirror.v)) atom_max_release_gpu(&p.st->dma_mirror.v, dh);
    if (h > ld_relaxed_gpu(&p.st->head_mirror.v)) atom_max_release_gpu(&p.st->head_mirror.v, h);
    if (sp) st_release_gpu(&p.st->stop.v, 1ull);
    st_relaxed_gpu(&p.st->poll_time.v, globaltimer());
    atomicExch(&p.st->poll_lock.v, 0ull);
  }

  // Nothing claimable: poll, fetch, decide exit, back off. False = leave.
  __device__ __forceinline__ bool idle_step() {
    const int m = serve_mail(false);
    if (m != 0) return m > 0;
    const u64 c0 = clock64();
    u32 leave = 0;
    if (lane == 0) {
      const u64 now = globaltimer();
      if (aborted() || ld_relaxed_gpu(&p.st->stop.v) != 0) {
        leave = 1;
      } else if (drain) {
        const u64 dn = ld_relaxed_gpu(&p.st->ops_done.v);
        if (dn >= ld_relaxed_gpu(&p.st->head_mirror.v) - p.base) {
          leave = 1;
        } else if (blockIdx.x == 0) {
          // drain watchdog: published work is left but nothing was handed out for idle_exit_ns
          const u64 act = ld_relaxed_gpu(&p.st->activity.v);
          if (now > act && now - act > p.idle_exit_ns) {
            raise_error(p.st, p.hctl, GPUOS_ETIMEDOUT, p.base + dn);
            leave = 1;
          }
        }
      } else {
        poll_host(now);
        if (blockIdx.x == 0) {
          const u64 act = ld_relaxed_gpu(&p.st->activity.v);
          const u64 hm = ld_relaxed_gpu(&p.st->head_mirror.v);
          const u64 nx = ld_relaxed_gpu(&p.st->next_op.v);
          const u64 dn = ld_relaxed_gpu(&p.st->ops_done.v);
          const u64 upto = nx < hm ? nx : hm;
          if (now > act && now - act > p.idle_exit_ns && nx >= hm && dn >= upto - p.base) {
            st_release_gpu(&p.st->stop.v, 2ull);
            p.hctl->exited_idle = 1u;
            fence_acq_rel_sys();
            leave = 1;
          }
        }
      }
    }
    if (bcast32(leave)) return false;
    const bool fetch = help_fetch();
    if (!fetch) {
      if (lane == 0) {
        backoff = backoff == 0 ? 32 : (backoff * 2 > p.backoff_ns ? p.backoff_ns : backoff * 2);
        __nanosleep(backoff);
      }
    }
    if (lane == 0) idle_cyc += clock64() - c0;
    return true;
  }

  // Tries to claim the FOLLOW ops after c as one run.
  __device__ __forceinline__ void try_extend(u64 c) {
    u64 hm = 0;
    if (lane == 0) hm = ld_acquire_gpu(&p.st->head_mirror.v);
    hm = bcast(hm);
    const u64 id = c + 1 + (u64)lane;
    bool ok = false;
    if (lane < 31 && id < hm) {
      const u64 h = hdr_of(id);
      ok = hdr_tag(h) == id + 1 && hdr_follow(h) && hdr_items(h) == 1;
    }
    const unsigned m = __ballot_sync(FULLMASK, ok);
    const u32 r = (u32)__ffs(~m) - 1u;
    if (r == 0) return;
    u32 won = 0;
    if (lane == 0) won = atomicCAS(&p.st->next_op.v, c + 1, c + 1 + r) == c + 1;
    if (bcast32(won)) {
      // each lane stages the descriptor whose tag it read with acquire ordering
      if ((u32)lane < r) {
        const uint4* src = reinterpret_cast<const uint4*>(ent(id));
        uint4* dst = reinterpret_cast<uint4*>(&S->stage[lane]);
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __ldcg(src + j);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = v[j];
      }
      __syncwarp();
      run_first = c + 1;
      run_next = c + 1;
      run_end = c + 1 + r;
    }
  }

  // 0 error, 1 emitted here, 2 posted to the CTA running its unfinished dependency.
  __device__ __forceinline__ int emit_single(u64 c, u32 claim, const RingEntry* staged = nullptr,
                                             bool handoff = false) {
    u64 d0 = 0, d1 = 0;
    if (lane == 0) {
      const RingEntry* e = staged ? staged : ent(c);
      d0 = e->dep0;
      d1 = e->dep1;
    }
    d0 = bcast(d0);
    d1 = bcast(d1);
    int ho = HO_NONE;
    if (handoff) {
      ho = try_handoff(c, d0, d1);
      if (ho == HO_POSTED) return 2;
      held = c + 1;  // dependants may be posted here from now on
      set_owner(c);
    }
    if (ho != HO_READY && !wait_deps(c, d0, d1)) return 0;
    if (!emit(c, 0, 1, claim, staged)) return 0;
    note_single(c);
    set_owner(c);
    if (handoff && !release_held()) return 0;
    return 1;
  }

  // -1 error, 0 nothing to join, 1 emitted an item of the open large op.
  __device__ __forceinline__ int try_join() {
    u32 valid = 0, item = 0, n = 0;
    u64 bid = 0;
    if (lane == 0) {
      const u64 w = ld_relaxed_gpu(&p.st->big.v);
      const u64 cur = w >> 24, cnt = w & BIG_COUNT_MASK;
      if (cur != 0) {
        const u64 h = hdr_of(cur - 1);
        if (hdr_tag(h) == cur && cnt < hdr_items(h)) {
          // a large op's items are taken with a shorter look-ahead than single
          // ops, so that no CTA holds items of it long before they run
          while ((unsigned)k - S->ncomp >= LOOKAHEAD_BIG) __nanosleep(20);
          const u64 v = atomicAdd(&p.st->big.v, 1ull);
          const u64 op1 = v >> 24, k2 = v & BIG_COUNT_MASK;
          const u64 h2 = (op1 == cur) ? h : (op1 ? hdr_of(op1 - 1) : 0ull);
          if (op1 != 0 && hdr_tag(h2) == op1 && k2 < hdr_items(h2)) {
            valid = 1;
            bid = op1 - 1;
            item = (u32)k2;
            n = (u32)hdr_items(h2);
          }
        }
      }
    }
    if (!bcast32(valid)) return 0;
    bid = bcast(bid);
    item = bcast32(item);
    n = bcast32(n);
    if (dep_ok != bid + 1) {
      u64 d0 = 0, d1 = 0;
      if (lane == 0) {
        d0 = ent(bid)->dep0;
        d1 = ent(bid)->dep1;
      }
      if (!wait_deps(bid, bcast(d0), bcast(d1))) return -1;
      dep_ok = bid + 1;
    }
    return emit(bid, item, n, CLAIM_BIG) ? 1 : -1;
  }

  // Opens the large op b once the previous large op has no items left.
  // -1 error, 0 not yet, 1 opened (item 0 emitted).
  __device__ __forceinline__ int try_install(u64 b) {
    u32 won = 0;
    if (lane == 0) {
      const u64 prev = ent(b)->prev_big;
      const u64 w = ld_relaxed_gpu(&p.st->big.v);
      const u64 cur = w >> 24, cnt = w & BIG_COUNT_MASK;
      bool free_ = false;
      if (cur == prev) {
        if (cur == 0) {
          free_ = true;
        } else {
          const u64 h = hdr_of(cur - 1);
          const u64 n = hdr_tag(h) == cur ? hdr_items(h) : 0;
          free_ = cnt >= n;
        }
      }
      if (free_) won = atomicCAS(&p.st->big.v, w, ((b + 1) << 24) | 1ull) == w;
      // progress watchdog: the open word must keep changing while we wait
      const u64 now = globaltimer();
      if (!won) {
        if (w != pend_word) {
          pend_word = w;
          pend_t = now;
        } else if (now - pend_t > p.timeout_ns) {
          raise_error(p.st, p.hctl, GPUOS_ETIMEDOUT, b);
        }
      }
    }
    if (!bcast32(won)) return aborted_b() ? -1 : 0;
    const u64 h = bcast(lane == 0 ? hdr_of(b) : 0ull);
    u64 d0 = 0, d1 = 0;
    if (lane == 0) {
      d0 = ent(b)->dep0;
      d1 = ent(b)->dep1;
    }
    if (!wait_deps(b, bcast(d0), bcast(d1))) return -1;
    dep_ok = b + 1;
    return emit(b, 0, (u32)hdr_items(h), CLAIM_BIG) ? 1 : -1;
  }

  __device__ __forceinline__ bool aborted_b() const {
    u32 a = 0;
    if (lane == 0) a = aborted();
    return bcast32(a) != 0;
  }

  // Waits (idle-style, no timeout) until id's descriptor is in the device ring.
  __device__ __forceinline__ bool wait_fetched(u64 id, u64& h) {
    for (;;) {
      u64 hh = 0;
      if (lane == 0) hh = hdr_of(id);
      hh = bcast(hh);
      if (hdr_tag(hh) == id + 1) {
        h = hh;
        return true;
      }
      if (!idle_step()) return false;
    }
  }

  // -1 leave, 0 idle, 1 did work, 2 retry at once.
  __device__ __forceinline__ int try_claim() {
    u64 c = 0, hm = 0;
    if (lane == 0) {
      c = ld_relaxed_gpu(&p.st->next_op.v);
      hm = ld_acquire_gpu(&p.st->head_mirror.v);
    }
    c = bcast(c);
    hm = bcast(hm);
    if (c >= hm) return 0;
    u64 h = bcast(lane == 0 ? hdr_of(c) : 0ull);
    if (hdr_tag(h) != c + 1) return help_fetch() ? 2 : 0;
    if (hdr_follow(h) && !is_local(c - 1)) {
      u32 ready = 0;
      if (lane == 0) ready = ld_acquire_gpu(&p.done[(c - 1) & p.mask]) >= c;
      if (!bcast32(ready)) return 0;  // the CTA that runs c - 1 is expected to take c
    }
    // claim, and read the peeked entry in the same round trip (lane 0 read its
    // tag with acquire ordering above; the warp barrier orders the other lanes)
    __syncwarp();
    u64 c2 = 0;
    uint4 chunk = uint4{0, 0, 0, 0};
    if (lane == 0) {
      // Near the head, claims take the peeked id by CAS: none runs ahead of
      // what the host published, and a FOLLOW op is left to its predecessor's
      // CTA. A drained session's head is fixed, so once this CTA has lost a
      // CAS race it claims by atomicAdd there too (a claim past the head is
      // simply empty); CAS contention would otherwise serialise the last
      // few hundred claims.
      if ((drain && contended && !hdr_follow(h)) || hm - c > 2ull * p.grid + 64ull) {
        c2 = atomicAdd(&p.st->next_op.v, 1ull);
      } else {
        c2 = atomicCAS(&p.st->next_op.v, c, c + 1) == c ? c : ~0ull;
        if (c2 == ~0ull) contended = true;
      }
    }
    if (lane < 8) chunk = __ldcg(reinterpret_cast<const uint4*>(ent(c)) + lane);
    if (lane == 0 && c2 != ~0ull) st_relaxed_gpu(&p.st->activity.v, globaltimer());
    c2 = bcast(c2);
    if (c2 == ~0ull) return 2;
    if (drain && c2 >= hm) return 0;
    ++claimed;
    backoff = 0;
    if (c2 != c && drain) {
      // A drained session's entries were all in the device ring before launch:
      // the tag, the dependencies and the entry come in one round trip.
      if (lane < 8) chunk = __ldcg(reinterpret_cast<const uint4*>(ent(c2)) + lane);
      const u64 h2 = __shfl_sync(FULLMASK, (u64)chunk.x | ((u64)chunk.y << 32), 0);
      if (hdr_tag(h2) == c2 + 1) {
        if (hdr_items(h2) > 1) {
          pending = c2 + 1;
          pend_word = ~0ull;
          return 1;
        }
        c = c2;  // continue below as if c2 had been the peeked op
        h = h2;
      }
    }
    if (c2 != c) {
      if (!wait_fetched(c2, h)) return -1;
      if (hdr_items(h) > 1) {
        pending = c2 + 1;
        pend_word = ~0ull;
        return 1;
      }
      const int r = emit_single(c2, CLAIM_SHARED, nullptr, true);
      if (r == 0) return -1;
      if (r == 1) try_extend(c2);
      return 1;
    }
    if (hdr_items(h) > 1) {
      pending = c2 + 1;
      pend_word = ~0ull;
      return 1;
    }
    // dependencies straight from the entry in registers (dep0: lane 0, dep1: lane 1)
    const u64 d0 = __shfl_sync(FULLMASK, (u64)chunk.z | ((u64)chunk.w << 32), 0);
    const u64 d1 = __shfl_sync(FULLMASK, (u64)chunk.x | ((u64)chunk.y << 32), 1);
    const int ho = try_handoff(c, d0, d1);
    if (ho == HO_POSTED) return 1;
    held = c + 1;  // dependants may be posted here from now on
    set_owner(c);
    if (ho != HO_READY && !wait_deps(c, d0, d1)) return -1;
    if (!emit(c, 0, 1, CLAIM_SHARED, nullptr, true, chunk)) return -1;
    note_single(c);
    if (!release_held()) return -1;
    try_extend(c);
    return 1;
  }

  __device__ __forceinline__ void run() {
    for (;;) {
      if ((++iters & 63) == 0 && aborted_b()) break;
      if (run_next < run_end) {
        const u64 c = run_next;
        if (!emit_single(c, CLAIM_RUN, &S->stage[c - run_first])) break;
        ++runops;
        ++run_next;
        if (run_next == run_end) try_extend(c);
        backoff = 0;
        continue;
      }
      {
        const int m = serve_mail(true);
        if (m < 0) break;
        if (m > 0) continue;
      }
      if (!throttle(LOOKAHEAD)) break;
      if (pending) {
        const int r = try_install(pending - 1);
        if (r < 0) break;
        if (r > 0) {
          pending = 0;
          backoff = 0;
          continue;
        }
        const int j = try_join();
        if (j < 0) break;
        if (j > 0) continue;
        if (!idle_step()) break;
        continue;
      }
      const int j = try_join();
      if (j < 0) break;
      if (j > 0) {
        backoff = 0;
        continue;
      }
      const int c = try_claim();
      if (c < 0) break;
      if (c > 0) continue;
      if (!idle_step()) break;
    }
    emit_exit();
    if (lane == 0) {
      CtaStats& cs = p.stats[blockIdx.x];
      cs.ops_claimed = claimed;
      cs.run_ops = runops;
      cs.idle_cycles = idle_cyc;
      cs.dep_cycles = dep_cyc;
      cs.fetch_descs = fetched;
    }
  }
};

// ------------------------------------------------------------------ publisher (one lane)
// Publishes every item the compute warps have finished, in batches: one
// device-scope fence makes the batch's outputs visible before its completion
// words, one system-scope fence before the host completion entries.
__device__ __forceinline__ bool mbar_test(unsigned long long* bar, unsigned int parity) {
  unsigned int ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ void publisher(const KParams& p, Smem* S) {
  const bool trace = (p.flags & KF_TRACE) != 0;
  u64 items = 0, smin = ~0ull, smax = 0;
  const u32 sm = smid();
  bool leave = false;
  for (u64 k = 0; !leave;) {
    {
      const u32 slot = (u32)(k % FIFO);
      while (!mbar_try_wait(&S->done_bar[slot], (u32)((k / FIFO) & 1))) {
      }
    }
    u32 m = 1;  // finished slots k .. k+m-1
    while (m < FIFO && mbar_test(&S->done_bar[(k + m) % FIFO], (u32)(((k + m) / FIFO) & 1))) ++m;
    u32 last_mask = 0, nwork = 0;
    fence_acq_rel_gpu();
    for (u32 j = 0; j < m; ++j) {
      const Slot& s = S->slot[(k + j) % FIFO];
      if (s.kind == SLOT_EXIT) {
        leave = true;
        break;
      }
      ++nwork;
      const u64 id = s.id;
      const u64 idx = id & p.mask;
      bool last = true;
      if (s.nitems > 1) {
        const u32 old = atom_add_acq_rel_gpu(&p.tiles_done[idx], 1u);
        last = (old + 1 == s.nitems);
        if (last) p.tiles_done[idx] = 0u;
      }
      if (s.t_start < smin) smin = s.t_start;
      if (s.t_end > smax) smax = s.t_end;
      if (trace) {
        gpuos_trace_rec* tr = &p.trace[idx];
        if (s.nitems == 1) {
          tr->t_start = s.t_start;
          tr->t_end = s.t_end;
          tr->items = 1;
        } else {
          atomicMin(reinterpret_cast<unsigned long long*>(&tr->t_start), s.t_start);
          atomicMax(reinterpret_cast<unsigned long long*>(&tr->t_end), s.t_end);
          atomicAdd(&tr->items, 1u);
        }
        if (last) {
          tr->cta = blockIdx.x;
          tr->smid = sm;
          tr->claim = s.claim;
          tr->id = id + 1;
        }
      }
      if (last) {
        // A single-item op's outputs are covered by the batch fence above
        // (fence + relaxed store is a release pattern). The last item of a
        // large op acquired the other items' outputs through the counter,
        // so its store itself must release them.
        if (s.nitems > 1)
          st_release_gpu(&p.done[idx], id + 1);
        else
          st_relaxed_gpu(&p.done[idx], id + 1);
        last_mask |= 1u << j;
      }
    }
    if (last_mask) {
      atomicAdd(&p.st->ops_done.v, (u64)__popc(last_mask));
      fence_acq_rel_sys();
      for (u32 j = 0; j < nwork; ++j) {
        if (last_mask & (1u << j)) {
          const u64 id = S->slot[(k + j) % FIFO].id;
          st_relaxed_sys_u64(&p.hdone[id & p.mask], id + 1);
        }
      }
    }
    for (u32 j = 0; j < nwork; ++j) mbar_arrive(&S->free_bar[(k + j) % FIFO]);
    items += nwork;
    k += nwork;
  }
  if (items) {
    atomicMin(&p.st->span_start.v, smin);
    atomicMax(&p.st->span_end.v, smax);
  }
  p.stats[blockIdx.x].items = items;
}

// ------------------------------------------------------------------ compute warps
__device__ void compute(const KParams& p, Smem* S, WarpSmem* W, int warp, int lane) {
  Cx cx;
  cx.tid = threadIdx.x - 64;
  cx.nthr = NCW * 32;
  cx.warp = warp - 2;
  cx.nwarps = NCW;
  cx.lane = lane;
  cx.bar = 1;
  cx.part = S->part;
  cx.ws = W + (warp - 2);
  cx.st = p.st;
  cx.hctl = p.hctl;
  cx.id = 0;
  cx.flags = p.flags;
  cx.rot = &S->rot;
  const bool leader = cx.tid == 0;
  for (u64 k = 0;; ++k) {
    const u32 slot = (u32)(k % FIFO);
    const u32 par = (u32)((k / FIFO) & 1);
    while (!mbar_try_wait(&S->full_bar[slot], par)) {
    }
    Slot& s = S->slot[slot];
    if (s.kind == SLOT_EXIT) {
      if (leader) mbar_arrive(&S->done_bar[slot]);
      break;
    }
    const u64 t0 = leader ? globaltimer() : 0ull;
    OpEnv env{p.st, p.hctl, p.timeout_ns, s.id};
    cx.id = s.id;
    run_item(s.e, s.item, p.elem_chunk, p.row_chunk, cx, env);
    cx_sync(cx);
    if (leader) {
      s.t_start = t0;
      s.t_end = globaltimer();
      S->ncomp = (unsigned)(k + 1);
      mbar_arrive(&S->done_bar[slot]);
    }
  }
}

// Dynamic shared memory: the scheduling block, then one staging area per compute warp.
constexpr size_t SMEM_HDR = (sizeof(Smem) + 127) / 128 * 128;
constexpr size_t PERSISTENT_SMEM = SMEM_HDR + NCW * sizeof(WarpSmem);
static_assert(PERSISTENT_SMEM <= 227 * 1024, "fits one SM");

__global__ void __launch_bounds__(NTHREADS, 1) gpuos_persistent_kernel(const __grid_constant__ KParams p) {
  extern __shared__ __align__(128) unsigned char dsm[];
  Smem& S = *reinterpret_cast<Smem*>(dsm);
  WarpSmem* W = reinterpret_cast<WarpSmem*>(dsm + SMEM_HDR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    S.ncomp = 0;
    S.rot.cols = 0;
    for (int i = 0; i < FIFO; ++i) {
      mbar_init(&S.full_bar[i], 1);
      mbar_init(&S.done_bar[i], 1);
      mbar_init(&S.free_bar[i], 1);
    }
    for (int wi = 0; wi < NCW; ++wi) {
      W[wi].seq = 0;
      for (int j = 0; j < WS_STAGES; ++j) mbar_init(&W[wi].bar[j], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {
    Control c(p, &S, lane);
    c.run();
  } else if (warp == 1) {
    if (lane == 0) publisher(p, &S);
  } else {
    compute(p, &S, W, warp, lane);
  }
}

__global__ void gpuos_reset_kernel(const KParams p, u64 head, u64 big_init) {
  const u64 tid = (u64)blockIdx.x * blockDim.x + threadIdx.x;
  const u64 nth = (u64)gridDim.x * blockDim.x;
  if (tid == 0) {
    DevState* st = p.st;
    st->next_op.v = p.base;
    st->fetch_next.v = p.fetched_upto > p.base ? p.fetched_upto : p.base;
    st->dma_mirror.v = st->fetch_next.v;
    st->head_mirror.v = head;
    st->big.v = big_init;
    st->poll_lock.v = 0;
    st->poll_time.v = 0;
    st->stop.v = 0;
    st->abort_.v = 0;
    st->ops_done.v = 0;
    st->err.v = 0;
    st->activity.v = globaltimer();
    st->span_start.v = ~0ull;
    st->span_end.v = 0;
  }
  for (u64 i = tid; i <= p.mask; i += nth) {
    p.tiles_done[i] = 0u;
    if (p.flags & KF_TRACE) {
      gpuos_trace_rec r;
      r.id = 0;
      r.t_start = ~0ull;
      r.t_end = 0;
      r.cta = 0;
      r.smid = 0;
      r.items = 0;
      r.claim = 0;
      p.trace[i] = r;
    }
  }
  for (u64 i = tid; i < p.grid; i += nth) {
    CtaStats z = {};
    p.stats[i] = z;
    if (p.mctl) {
      p.mctl[i].tail = 0;
      p.mctl[i].head = 0;
    }
  }
  if (p.mbox)
    for (u64 i = tid; i < (u64)p.grid * MAILBOX; i += nth) p.mbox[i] = 0;
}

int launch_session(const KParams& p, u64 head, u64 big_init, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  gpuos_reset_kernel<<<64, 256, 0, s>>>(p, head, big_init);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  static bool attr_set = false;  // per process; the attribute is per function, not per device
  if (!attr_set) {
    e = cudaFuncSetAttribute(gpuos_persistent_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PERSISTENT_SMEM);
    if (e != cudaSuccess) return (int)e;
    attr_set = true;
  }
  gpuos_persistent_kernel<<<p.grid, NTHREADS, PERSISTENT_SMEM, s>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace gpuos_impl
