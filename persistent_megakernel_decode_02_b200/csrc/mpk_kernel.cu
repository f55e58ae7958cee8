// Persistent decode megakernel for B200 (sm_100a).
//
// One launch runs every decoding iteration of a run ("Mirage Persistent
// Kernel: Fusing Multi-GPU LLM Inference into One Kernel Launch", section
// "How MPK Works": a persistent kernel stays resident for the whole inference
// loop; each fused operation is a task of a task graph).  Blocks take one of
// two roles, split as num_workers + num_schedulers/4 = #SMs (same section):
//
//  * scheduler blocks: 4 scheduler warps each; every lane of a scheduler warp
//    owns one worker and pushes that worker's task entries, in graph order,
//    into its global-memory queue.  Dispatch of operation g is gated on the
//    completion event of operation g - lookahead, so queues run a bounded
//    distance ahead of execution ("工作机制": tasks are assigned to workers by
//    schedulers on the GPU).
//  * worker blocks (one per SM): warp 0 is the producer; it pops task entries
//    and streams the task's weight rows into a ring of shared-memory stages with
//    1-D bulk (TMA) copies, running ahead into the NEXT tasks while the
//    consumers still work — weights do not depend on activations, so the next
//    layer's weights load while the current layer computes (MPK blog excerpt,
//    "Why MPK?": software pipelining across layers).  Warps 1..8 are consumers:
//    they wait for the task's dependency event, compute, and release-increment
//    the task's completion event.
//
// Every device wait is bounded by a %globaltimer deadline; on expiry the
// waiter records the failure in the status block and all roles return.  Only
// one elected thread of a consumer group ever waits, and its outcome is shared
// through shared memory behind a named barrier that every consumer reaches, so
// an abort can never leave threads stuck in a hardware barrier.

#include <cuda_runtime.h>
#include <stdint.h>

#include "mpk_internal.h"
#include "mpk_ptx.cuh"

namespace mpk {

// ------------------------------------------------------------------ shared memory
struct AttnScratch {
  float qs[MAX_G * MAX_D / 2];                   // normalised, rotated queries (G*d <= 512)
  uint16_t ks[MAX_D];                            // this position's k (bf16)
  uint16_t vs[MAX_D];                            // this position's v (bf16)
  float wm[CONSUMER_WARPS][MAX_G][2];            // per-warp running (max, sum)
  float wacc[CONSUMER_WARPS][MAX_G * MAX_D / 2]; // per-warp unnormalised outputs
  float4 xs[CONSUMER_WARPS * 32];                // tensor-core path: partial scores exchanged by a tile's two warps
};
static_assert(MAX_G * MAX_D / 2 >= 512, "attention scratch");
static_assert(CONSUMER_WARPS * (MAX_G * MAX_D / 2) >= 2 * (MAX_G / 2) * MAX_SPLIT_CHUNKS + MAX_G / 2,
              "the split merge's chunk weights and sums fit the per-warp output scratch (G <= 4)");
static_assert(sizeof(AttnScratch) >= sizeof(float) * MAX_GCHUNK * (MAX_G / 2) * (MAX_D + 2),
              "the group merge gathers every chunk partial of a kv head into the attention scratch");

struct __align__(128) Smem {
  uint8_t ring[NSTAGES][STAGE_BYTES];
  union {
    AttnScratch a;
    struct {
      float hs[MAX_K];                           // GEMV input vector (fp32)
      float xs[MAX_XS];                          // residual rows of the task
    } g;
  } u;
  float ss[CONSUMER_WARPS];
  unsigned long long bestk[CONSUMER_WARPS];
  unsigned long long fifo[TASK_FIFO];
  uint64_t full[NSTAGES];
  uint64_t empty[NSTAGES];
  uint64_t fifo_full[TASK_FIFO];
  uint64_t fifo_empty[TASK_FIFO];
  unsigned long long cur_entry;
  unsigned long long fifo_t[TASK_FIFO];          // profiling: first weight stage issued
  unsigned long long t_pro, t_data;              // profiling: prologue done, first stage ready
  unsigned long long t_stall, t_last;            // profiling: time waited for stages, last stage ready
  unsigned long long t_loop;                     // profiling: every consumer warp done with its rows
  int32_t last;     // last-arrival flag
  int32_t attn_s;   // fused QKV + attention: position of the request (-1: inactive), read in the prologue
  unsigned long long h_key;  // (iteration, op, segment) whose input vector hs holds (~0: none)
  float2 rope_row[MAX_D / 2];                    // its RoPE (cos, sin) row
  // tensor-core path
  uint64_t acc_full[NSLOT_MAX];                  // accumulator slot b holds a finished row block
  uint64_t acc_empty[NSLOT_MAX];                 // slot b has been read (one arrival per epilogue warp)
  uint64_t bfree;                                // the MMAs of a pass are done with the input rows
  uint32_t bfn;                                  // completed phases of bfree (read and advanced by consumer thread 0)
  uint64_t bload;                                // the published input rows of a pass have landed
  uint32_t bload_n;                              // completed phases of bload (the MMA-issuing thread's)
  uint64_t fin_bar;                              // drain of outstanding MMAs before exit
  uint32_t tmem_base;                            // tensor-memory address of the accumulators
  int32_t blast;                                 // this task finishes the current row block
  float brinv[MAX_BATCH];                        // per-request RMSNorm factor of the task's input
  float bss[2][4][MAX_BATCH];                    // per block parity, epilogue warp, request: sums of squares
  unsigned long long bbest[4][MAX_BATCH];        // LM head: per epilogue warp and request (value, index) maxima
};
static_assert(NSTB < NSTAGES && 2 * MAX_PREFILL * MAX_D * 2 <= STAGE_BYTES,
              "a prefill attention task's k/v rows fit the stage the tensor-core path keeps for its inputs");
static_assert((NSTAGES - NSTB) * STAGE_BYTES + sizeof(((Smem*)nullptr)->u) >= B_INPUT_BYTES,
              "the batch input rows fit in the stages the ring leaves free and the scratch after them");

// ------------------------------------------------------------------ status / waits
__device__ __forceinline__ bool aborted(const Graph& g) {
  if (ld_volatile_i32(&g.status->code) != 0) return true;
  return false;
}

__device__ __noinline__ void record_error_at(Status* st, int code, int where, int op, int task, int worker,
                                             int iter, uint32_t observed, uint32_t expected) {
  if (atomicCAS(&st->code, 0, code) == 0) {
    st->where = where;
    st->op = op;
    st->task = task;
    st->worker = worker;
    st->iter = iter;
    st->observed = observed;
    st->expected = expected;
    __threadfence();
  }
}

__device__ __forceinline__ void record_error(const Graph& g, int code, int where, int op, int task, int worker,
                                             int iter, uint32_t observed, uint32_t expected) {
  record_error_at(g.status, code, where, op, task, worker, iter, observed, expected);
}

// Polls the host abort flag (mapped memory, slow) only now and then.
__device__ __forceinline__ bool check_stop(const Graph& g, uint64_t t0, uint32_t it, int where, int op,
                                           int task, int worker, int iter, uint32_t obs, uint32_t exp) {
  if ((it & 255u) != 255u) return false;
  if (aborted(g)) return true;
  if ((it & 0xFFFFu) == 0xFFFFu && g.abort_flag != nullptr && *g.abort_flag != 0) {
    record_error(g, -10 /*ABORTED*/, where, op, task, worker, iter, obs, exp);
    return true;
  }
  if (globaltimer() - t0 > g.timeout_ns) {
    record_error(g, -9 /*TIMEOUT*/, where, op, task, worker, iter, obs, exp);
    return true;
  }
  return false;
}

// Wait until *ctr >= target (wrap-safe).  Returns false on abort/timeout.
__device__ bool wait_counter(const Graph& g, const uint32_t* ctr, uint32_t target, int where, int op,
                             int task, int worker, int iter) {
  uint32_t v = ld_acquire(ctr);
  if ((int32_t)(v - target) >= 0) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    v = ld_acquire(ctr);
    if ((int32_t)(v - target) >= 0) return true;
    if (check_stop(g, t0, it, where, op, task, worker, iter, v, target)) return false;
  }
}

__device__ bool wait_mbar(const Graph& g, uint64_t* bar, uint32_t parity, int where, int worker) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (check_stop(g, t0, it, where, -1, -1, worker, -1, parity, 0)) return false;
  }
}

// Version tag of the values op `writer` writes in iteration `iter`.
__device__ __forceinline__ uint32_t vtag(const Graph& g, uint32_t iter, int writer) {
  return iter * (uint32_t)g.nops + (uint32_t)writer + 1u;
}

// Value of a tagged element once it carries `tag` (the word already loaded is
// tried first).  False on abort or timeout (the value is then meaningless).
__device__ __noinline__ bool poll_tagged(const Graph& g, const uint64_t* p, uint64_t w, uint32_t tag, float& v,
                                         int op, int worker, int iter) {
  if (word_tag(w) == tag) {
    v = word_value(w);
    return true;
  }
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    w = ld_tagged(p);
    if (word_tag(w) == tag) {
      v = word_value(w);
      return true;
    }
    if (check_stop(g, t0, it, 11, op, -1, worker, iter, word_tag(w), tag)) {
      v = 0.f;
      return false;
    }
  }
}

// The word at p once it carries `tag`; on abort or timeout the last word read
// (its tag differs, which the caller checks).  Takes no address of the
// caller's variables, so their arrays stay in registers.
__device__ __noinline__ uint64_t poll_word(const Graph& g, const uint64_t* p, uint32_t tag, int op, int worker,
                                           int iter) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    const uint64_t w = ld_tagged(p);
    if (word_tag(w) == tag) return w;
    if (check_stop(g, t0, it, 11, op, -1, worker, iter, word_tag(w), tag)) return w;
  }
}

// n consecutive tagged elements into fp32: all loads issued first, stragglers
// polled.  Returns false on abort or timeout.
template <int N>
__device__ __forceinline__ bool load_tagged(const Graph& g, const uint64_t* p, uint32_t tag, float* out, int op,
                                            int worker, int iter) {
  uint64_t w[N];
#pragma unroll
  for (int e = 0; e < N; ++e) w[e] = ld_tagged(p + e);
  bool ok = true;
#pragma unroll
  for (int e = 0; e < N; ++e) {
    if (word_tag(w[e]) == tag) out[e] = word_value(w[e]);
    else ok &= poll_tagged(g, p + e, w[e], tag, out[e], op, worker, iter);
  }
  return ok;
}

// A batch of tagged words, all loaded before any is looked at (so a prologue
// costs one memory round trip, not one per load), settled until every word
// that valid(u) selects carries `tag`.  While one is not current, that word
// alone is polled until it is, then the whole batch is read again in one
// round trip.  The batch is reloaded after every wait, so none of it stays
// live across the waiting call.  addr(u) is the address of word u.  False on
// abort or timeout.
template <int N, typename Addr, typename Valid>
__device__ __forceinline__ bool settle_tagged(const Graph& g, uint64_t (&w)[N], Addr addr, Valid valid, uint32_t tag,
                                              int op, int worker, int iter) {
  for (;;) {
    int bad = -1;
#pragma unroll
    for (int u = 0; u < N; ++u)
      if (valid(u) && word_tag(w[u]) != tag) bad = u;
    if (bad < 0) return true;
    const uint64_t x = poll_word(g, addr(bad), tag, op, worker, iter);
    if (word_tag(x) != tag) {
#pragma unroll
      for (int u = 0; u < N; ++u) w[u] = 0ull;
      return false;
    }
#pragma unroll
    for (int u = 0; u < N; ++u) w[u] = valid(u) ? ld_tagged(addr(u)) : 0ull;
  }
}

// ------------------------------------------------------------------ task geometry
// Rows [row0, row1) of group g that task `task` computes (groups split the
// tasks evenly; N is the row count of one group).
// A split residual projection (ksplit > 1) has nb = ntasks / ksplit row
// blocks; task t computes reduction segment t / nb of row block t % nb
// (consecutive tasks share a segment, so a worker claiming several keeps its
// input segment).
__device__ __forceinline__ void task_rows(const OpDesc& op, int task, int& g, int& row0, int& row1) {
  int tpg = op.ntasks / op.groups, t;
  if (op.ksplit > 1) {
    tpg /= op.ksplit;
    g = 0;
    t = task % tpg;
  } else {
    g = task / tpg;
    t = task - g * tpg;
  }
  row0 = (int)(((long long)t * op.N) / tpg);
  row1 = (int)(((long long)(t + 1) * op.N) / tpg);
}

// First reduction element of the task's segment (0 without a split).
__device__ __forceinline__ int task_seg(const OpDesc& op, int task) {
  return op.ksplit > 1 ? task / (op.ntasks / op.ksplit) : 0;
}
__device__ __forceinline__ int task_koff(const OpDesc& op, int task) { return task_seg(op, task) * op.kseg; }

// Reduction length of one task (the segment length for a split projection).
__device__ __forceinline__ int task_k(const OpDesc& op) { return op.ksplit > 1 ? op.kseg : op.K; }

// Weight bytes of one task row in a stage (gate/up: both matrices).
__device__ __forceinline__ uint32_t stage_row_bytes(const OpDesc& op) {
  return (uint32_t)task_k(op) * 2u * (op.kind == TK_NORM_GEMV_SILU ? 2u : 1u);
}

__device__ __forceinline__ bool is_gemv(int kind) {
  return kind == TK_NORM_GEMV || kind == TK_GEMV_RESID || kind == TK_NORM_GEMV_SILU ||
         kind == TK_NORM_GEMV_ARGMAX || kind == TK_QKV_ATTN;
}

// The position and request of column r in iteration `iter`, and whether it is
// active.  Without prefill column r is request r, one position per
// iteration.  A prefill graph ingests its requests one after another: the
// iteration's request q is the one whose share of the run's iterations
// (ceil(remaining positions / R) each, in request order) holds `iter`, and
// column r is at q's position for that iteration plus r.
// In a persistent run this comes from the run-start state (nothing written
// during the run is read): per column (per request for prefill) the first
// position and the last it may reach, and for prefill the iterations before
// each request.
__device__ __forceinline__ bool request_at(const Graph& g, int r, uint32_t iter, int& s, int& q) {
  if (!g.prefill) {
    q = r;
    const int s0 = __ldcg(&g.ctl->step0[r]);
    s = s0 + (int)iter;
    return s0 >= 0 && s < __ldcg(&g.ctl->stop[r]);
  }
  q = 0;
  for (int i = 1; i < g.Rq; ++i)
    if (__ldcg(&g.ctl->cum[i]) <= iter) q = i;
  const int s0 = __ldcg(&g.ctl->step0[q]);
  s = s0 + (int)(iter - __ldcg(&g.ctl->cum[q])) * g.R + r;
  return s0 >= 0 && s < __ldcg(&g.ctl->stop[q]);
}

// The same from `step` itself, when every operation is its own launch (the
// launches order the updates): a prefill graph serves the first request
// that still has positions to go.
__device__ __forceinline__ bool request_active(const Graph& g, int r, int& s, int& q) {
  auto last_pos = [&](int rq) {
    int end = g.S - 1;
    if (g.step_end != nullptr) {
      const int e = __ldcg(g.step_end + rq);
      end = e < end ? e : end;
    }
    return end;
  };
  if (!g.prefill) {
    q = r;
    s = __ldcg(g.step + r);
    return s >= 0 && s < last_pos(r);
  }
  q = 0;
  int st = -1;
  for (int i = 0; i < g.Rq; ++i) {
    const int si = __ldcg(g.step + i);
    if (si >= 0 && si < last_pos(i)) {
      q = i;
      st = si;
      break;
    }
  }
  s = st + r;
  return st >= 0 && s < last_pos(q);
}

__device__ __forceinline__ bool request_state(const Graph& g, int r, uint32_t iter, int& s, int& q) {
  return g.op_by_op ? request_active(g, r, s, q) : request_at(g, r, iter, s, q);
}
__device__ __forceinline__ bool request_state(const Graph& g, int r, uint32_t iter, int& s) {
  int q;
  return request_state(g, r, iter, s, q);
}

// First position of the iteration's chunk of column r's request (column 0's
// position): prefill columns r' < r hold positions chunk0 .. s - 1.
__device__ __forceinline__ int chunk0(const Graph& g, int r, int s) { return s - (g.prefill ? r : 0); }

// Row of the split-K operation's cache, viewed as [rows, d], that holds
// position p of request q and kv head j; -1 when a paged cache's page table
// names no page of the cache there (the caller records the error).
__device__ __forceinline__ int kv_row(const Graph& g, const OpDesc& op, int q, int j, int p) {
  if (op.page == 0) return ((op.layer * g.Rq + q) * op.Hkv + j) * op.S + p;
  const int pg = __ldg(op.kv_pages + q * op.max_pages + p / op.page);
  if (pg < 0 || pg >= op.npages) return -1;
  return ((op.layer * op.npages + pg) * op.Hkv + j) * op.page + p % op.page;
}

// Positions [lo, hi) of chunk c of C of a split-K task over npos positions:
// an even split; with a paged cache the inner boundaries are rounded down to a
// multiple of the stage length PB, so that every stage but a chunk's last is
// whole (the chunks still cover 0..npos-1 once, the last one ends at npos).
__device__ __forceinline__ void chunk_bounds(const OpDesc& op, int c, int C, int npos, int& lo, int& hi) {
  lo = (int)(((long long)c * npos) / C);
  hi = (int)(((long long)(c + 1) * npos) / C);
  if (op.page > 0) {
    const int PB = STAGE_BYTES / (4 * op.d);
    lo = lo / PB * PB;
    if (c + 1 < C) hi = hi / PB * PB;
  }
}

// End of the stage that starts at position p of a split-K chunk ending at
// hi: PB positions on; with a paged cache up to the next multiple of PB (the
// page size is a multiple of PB, so no stage straddles two pages).
__device__ __forceinline__ int attn_stage_end(const OpDesc& op, int p, int hi, int PB) {
  const int e = op.page > 0 ? (p / PB + 1) * PB : p + PB;
  return e < hi ? e : hi;
}

// Locate global row `row` of a stacked multi-matrix operation.
__device__ __forceinline__ int seg_of(const OpDesc& op, int row) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < MAX_SEG; ++i)
    if (i < op.nseg && row >= op.seg_row0[i]) s = i;
  return s;
}

// Matrix row of group-local row `row` that lies in segment s.
__device__ __forceinline__ size_t seg_row(const OpDesc& op, int g, int s, int row) {
  return (size_t)g * op.grp_rows[s] + (size_t)(row - op.seg_row0[s]);
}

// ------------------------------------------------------------------ producer
// Issue the bulk copies of one stage: rows [r, r+n) of the op's row space.
__device__ void issue_stage(const OpDesc& op, int g, int r, int n, int koff, uint8_t* dst, uint64_t* bar,
                            uint64_t pol) {
  const uint32_t row_bytes = (uint32_t)op.K * 2u;
  if (op.ksplit > 1) {
    // one segment of each row: rows are strided in memory
    const uint32_t seg_bytes = (uint32_t)op.kseg * 2u;
    for (int i = 0; i < n; ++i)
      bulk_g2s(dst + (size_t)i * seg_bytes, op.W[0] + (size_t)(r + i) * op.K + koff, seg_bytes, bar, pol);
    return;
  }
  if (op.kind == TK_NORM_GEMV_SILU) {
    bulk_g2s(dst, op.W[0] + (size_t)r * op.K, row_bytes * n, bar, pol);
    bulk_g2s(dst + (size_t)op.rps * row_bytes, op.W_up + (size_t)r * op.K, row_bytes * n, bar, pol);
    return;
  }
  while (n > 0) {
    const int s = seg_of(op, r);
    const int seg_end = op.seg_row0[s + 1];
    const int cnt = min(n, seg_end - r);
    bulk_g2s(dst, op.W[s] + seg_row(op, g, s, r) * op.K, row_bytes * cnt, bar, pol);
    dst += (size_t)cnt * row_bytes;
    r += cnt;
    n -= cnt;
  }
}

// Prefetch rows [r, r+n) of a GEMV operation's weights into L2.
__device__ void prefetch_rows(const OpDesc& op, int g, int r, int n, int koff) {
  const uint32_t row_bytes = (uint32_t)op.K * 2u;
  if (op.ksplit > 1) {
    for (int i = 0; i < n; ++i) prefetch_l2(op.W[0] + (size_t)(r + i) * op.K + koff, (uint32_t)op.kseg * 2u);
    return;
  }
  if (op.kind == TK_NORM_GEMV_SILU) {
    prefetch_l2(op.W[0] + (size_t)r * op.K, row_bytes * n);
    prefetch_l2(op.W_up + (size_t)r * op.K, row_bytes * n);
    return;
  }
  while (n > 0) {
    const int s = seg_of(op, r);
    const int cnt = min(n, op.seg_row0[s + 1] - r);
    prefetch_l2(op.W[s] + seg_row(op, g, s, r) * op.K, row_bytes * cnt);
    r += cnt;
    n -= cnt;
  }
}

// The producer keeps a second cursor over the same task sequence that issues
// L2 prefetches for the weight bytes just beyond what the shared-memory ring
// will hold: [loaded + ring, loaded + ring + prefetch_bytes).  It peeks at
// queued entries without popping them (the scheduler never overwrites an entry
// that has not been popped), so HBM keeps streaming the next operations'
// weights while this worker waits on a dependency; bytes the ring itself is
// about to load are never requested twice.
struct PrefetchCursor {
  uint32_t q;              // queue index of the task the cursor is in
  int row;                 // next row of that task (-1: not started)
  bool done;               // reached the end of the queue
  bool have;               // e holds entry q (already popped, so not re-read)
  unsigned long long e;
  uint64_t pos;            // stream byte offset of (q, row)
};

// Chunk slots of the split-K attention operation: grid_dim = (Hkv, C, R),
// task (j, c, r) attends to chunk c of C of request r's positions.  The split
// of a request never depends on the other requests, so its results do not
// depend on the batch it shares an iteration with.
__device__ __forceinline__ bool attn_slot(const Graph& g, const OpDesc& op, int q, uint32_t iter, int& r, int& c,
                                          int& Cr) {
  (void)iter;
  r = q / op.C;
  c = q - r * op.C;
  Cr = op.C;
  return r < g.R;
}

// Ring stages a split-K attention task takes (the producer issues them, the
// consumer reads them): its chunk's cached positions, those below the
// iteration's chunk start (s; prefill: column 0's position), in blocks of
// STAGE_BYTES / (4 d).
__device__ __forceinline__ uint32_t attn_stages(const Graph& g, const OpDesc& op, int task, uint32_t iter) {
  int r, c, Cr, s;
  if (!attn_slot(g, op, task / op.Hkv, iter, r, c, Cr) || !request_state(g, r, iter, s)) return 0u;
  const int npos = s + 1, sc0 = chunk0(g, r, s);
  int lo, hi;
  chunk_bounds(op, c, Cr, npos, lo, hi);
  hi = hi < sc0 ? hi : sc0;
  const int PB = STAGE_BYTES / (4 * op.d);
  if (hi <= lo) return 0u;
  return op.page > 0 ? (uint32_t)((hi - 1) / PB - lo / PB + 1) : (uint32_t)((hi - lo + PB - 1) / PB);
}

// Producer side of a split-K attention task: the cached positions of its
// chunk, [lo, min(hi, chunk start)), into the ring, once the previous
// iteration's attention has released the operation (so those positions are in
// the cache).  A stage holds PB positions from p on: K in its first half, V in
// the second, each as d/64 boxes of [PB rows][64] bf16 (2-D tensor copies with
// 128-byte swizzle, box h holding dims 64h..64h+63).  The boxes always hold PB
// rows: those past the chunk's last position are loaded but never used.  The
// consumer takes exactly these stages.  False on abort or timeout.  Not
// inlined, so it adds nothing to the producer loop's registers.
__device__ __noinline__ bool attn_produce(Smem& sm, const Graph& g, const OpDesc& op, int task, uint32_t iter,
                                          uint32_t& pstage, int worker, uint64_t pol, int nr) {
  int r, c, Cr;
  if (!attn_slot(g, op, task / op.Hkv, iter, r, c, Cr)) return true;
  const int j = task % op.Hkv;
  int s, q;
  if (!request_state(g, r, iter, s, q)) return true;
  const int npos = s + 1, sc0 = chunk0(g, r, s);
  int lo, hi;
  chunk_bounds(op, c, Cr, npos, lo, hi);
  hi = hi < sc0 ? hi : sc0;
  if (hi <= lo) return true;
  if (iter > 0) {
    if (!wait_counter(g, g.events + (size_t)op.out_event * EVENT_STRIDE, iter * (uint32_t)op.out_trigger, 2, op.self,
                      task, worker, (int)iter))
      return false;
    // the cache rows were appended with ordinary stores: order them before
    // this thread's tensor copies read them
    fence_acq_rel_gpu();
    fence_proxy_async_global();
  }
  const int D = op.d, PB = STAGE_BYTES / (4 * D);
  for (int p = lo; p < hi; p = attn_stage_end(op, p, hi, PB)) {
    const int row = kv_row(g, op, q, j, p);  // rows < 2^31 (checked on the host)
    if (row < 0) {
      record_error(g, -11 /*DEVICE*/, 12, op.self, task, worker, (int)iter, (uint32_t)q, (uint32_t)p);
      return false;
    }
    const uint32_t slot = pstage % (uint32_t)nr;
    if (!wait_mbar(g, &sm.empty[slot], ((pstage / (uint32_t)nr) & 1u) ^ 1u, 3, worker)) return false;
    mbar_arrive_expect_tx(&sm.full[slot], (uint32_t)STAGE_BYTES);
    for (int h = 0; h < D / 64; ++h) {
      tma_load_2d(sm.ring[slot] + h * PB * 128, op.tmap_kc, h * 64, row, &sm.full[slot], pol);
      tma_load_2d(sm.ring[slot] + STAGE_BYTES / 2 + h * PB * 128, op.tmap_vc, h * 64, row, &sm.full[slot], pol);
    }
    ++pstage;
  }
  return true;
}

// Producer side of a tensor-core (batched) task; defined with the batched path.
template <int BW>
__device__ bool bproduce(Smem& sm, const Graph& g, const OpDesc& op, int task, uint32_t& pstage, int worker,
                         uint64_t pol, unsigned long long* t_issue);

// kSplit: the graph has split-K attention operations, whose K/V the producer
// streams (kernels without them leave the code out entirely); BW: the batch
// width of the tensor-core path.
template <bool kStandalone, bool kBatch, bool kSplit, int BW>
__device__ void producer_loop(Smem& sm, const Graph& g, int worker, uint32_t sa_iter, int sa_op) {
  constexpr int NR = kBatch ? NSTB : NSTAGES;  // weight stages of the ring
  const uint64_t pol = policy_evict_first();
  uint32_t qpos = 0, fpos = 0, pstage = 0;
  bool ok = true;
  uint32_t* qtail = g.q_tail + (size_t)worker * EVENT_STRIDE;
  uint32_t* qhead = g.q_head + (size_t)worker * EVENT_STRIDE;
  const unsigned long long* queue = g.queue + (size_t)worker * QUEUE_CAP;
  uint32_t tail_seen = 0;
  uint64_t ld_bytes = 0;
  PrefetchCursor pf{0u, -1, false, false, 0ull, 0ull};
  const uint64_t pf_dist = (kStandalone || kBatch) ? 0ull : (uint64_t)g.prefetch_bytes;
  constexpr uint64_t RING = (uint64_t)NR * STAGE_BYTES;

  auto prefetch_some = [&]() {
    const uint64_t lo = ld_bytes + RING, hi = lo + pf_dist;
    while (!pf.done && pf.pos < hi) {
      if (!pf.have) {
        // entries at or after the pop position are never overwritten
        if (pf.q >= tail_seen) {
          tail_seen = ld_acquire(qtail);
          if (pf.q >= tail_seen) return;
        }
        pf.e = __ldcg(queue + (pf.q % QUEUE_CAP));
        pf.have = true;
      }
      if (pf.e == QUEUE_TERMINATE) {
        pf.done = true;
        return;
      }
      if ((pf.e & 0xFFFFu) == TASK_CLAIM) {  // tasks claimed later: nothing to prefetch for yet
        ++pf.q;
        pf.row = -1;
        pf.have = false;
        continue;
      }
      const OpDesc& op = g.ops[(int)((pf.e >> 16) & 0xFFFFu)];
      int r0 = 0, r1 = 0, pg = 0;
      if (is_gemv(op.kind)) task_rows(op, (int)(pf.e & 0xFFFFu), pg, r0, r1);
      if (pf.row < 0) pf.row = r0;
      if (pf.row >= r1) {
        ++pf.q;
        pf.row = -1;
        pf.have = false;
        continue;
      }
      const uint32_t rb = stage_row_bytes(op);
      const int n = min(r1 - pf.row, max(1, (int)(65536u / rb)));
      if (pf.pos + (uint64_t)rb * n > lo) prefetch_rows(op, pg, pf.row, n, task_koff(op, (int)(pf.e & 0xFFFFu)));
      pf.row += n;
      pf.pos += (uint64_t)rb * n;
    }
  };

  int claim_op = -1;       // dynamic op whose tasks this worker is claiming (-1: none)
  uint32_t claim_iter = 0;
  while (true) {
    unsigned long long entry;
    if (kStandalone) {
      entry = (fpos == 0) ? pack_entry(sa_iter, (uint32_t)sa_op, blockIdx.x) : QUEUE_TERMINATE;
    } else if (claim_op >= 0) {
      // Claim the next task of the dynamic op, now that the ring has taken
      // the previous one.  Every worker claims until the counter passes the
      // task count; the last of those ntasks + W claims resets the counter,
      // whose slot serves iteration claim_iter + CLAIM_SLOTS next.
      const OpDesc& co = g.ops[claim_op];
      uint32_t* ctr = g.claims + ((size_t)(claim_iter % CLAIM_SLOTS) * g.nops + claim_op) * EVENT_STRIDE;
      const uint32_t c = atomicAdd(ctr, 1u);
      if (c >= (uint32_t)co.ntasks) {
        if (c == (uint32_t)(co.ntasks + g.num_workers - 1)) atomicExch(ctr, 0u);
        claim_op = -1;
        continue;
      }
      entry = pack_entry(claim_iter, (uint32_t)claim_op, c);
    } else {
      if (!wait_counter(g, qtail, qpos + 1, 2, -1, -1, worker, -1)) { ok = false; break; }
      entry = __ldcg(queue + (qpos % QUEUE_CAP));
      if (entry != QUEUE_TERMINATE && (entry & 0xFFFFu) == TASK_CLAIM) {
        ++qpos;
        st_release(qhead, qpos);
        claim_op = (int)((entry >> 16) & 0xFFFFu);
        claim_iter = (uint32_t)(entry >> 32);
        continue;
      }
      // a prefetch cursor that has not passed this task restarts at its first row
      if (pf.q < qpos || (pf.q == qpos && !pf.have)) {
        // the cursor is behind: restart it at this task (the stream offset of
        // its first row is the current load offset)
        pf.q = qpos;
        pf.row = -1;
        pf.have = true;
        pf.e = entry;
        pf.pos = ld_bytes;
      }
      ++qpos;
      st_release(qhead, qpos);
    }
    const uint32_t f = fpos % TASK_FIFO;
    if (!wait_mbar(g, &sm.fifo_empty[f], ((fpos / TASK_FIFO) & 1u) ^ 1u, 4, worker)) { ok = false; break; }
    sm.fifo[f] = entry;
    // profiling: the issue time of this task's first stage is stored before
    // the slot is published; it is overwritten below once the stage is issued
    // (the consumer reads it only at the end of the task).
    if (g.profiling) sm.fifo_t[f] = 0ull;
    mbar_arrive(&sm.fifo_full[f]);
    ++fpos;
    if (entry == QUEUE_TERMINATE) break;

    const int opi = (int)((entry >> 16) & 0xFFFFu);
    const int task = (int)(entry & 0xFFFFu);
    const OpDesc& op = g.ops[opi];
    if constexpr (kSplit) {
      if (op.kind == TK_ATTN) {
        if (!attn_produce(sm, g, op, task, (uint32_t)(entry >> 32), pstage, worker, pol, NR)) {
          ok = false;
          break;
        }
        continue;
      }
    }
    if (!is_gemv(op.kind)) continue;
    if constexpr (kBatch) {
      if (!bproduce<BW>(sm, g, op, task, pstage, worker, pol, g.profiling ? &sm.fifo_t[f] : nullptr)) {
        ok = false;
        break;
      }
      continue;
    }
    int grp, row0, row1;
    task_rows(op, task, grp, row0, row1);
    const uint32_t bytes_row = stage_row_bytes(op);
    const int koff = task_koff(op, task);
    for (int r = row0; r < row1; r += op.rps) {
      const int n = min(op.rps, row1 - r);
      const uint32_t slot = pstage % NSTAGES;
      const uint32_t par = ((pstage / NSTAGES) & 1u) ^ 1u;
      if (!mbar_try_wait(&sm.empty[slot], par)) {
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 0;; ++it) {
          if (pf_dist) prefetch_some();
          if (mbar_try_wait(&sm.empty[slot], par)) break;
          if (check_stop(g, t0, it, 3, opi, task, worker, -1, par, 0)) { ok = false; break; }
        }
        if (!ok) break;
      }
      if (g.profiling && r == row0) atomicExch(&sm.fifo_t[f], (unsigned long long)globaltimer());
      mbar_arrive_expect_tx(&sm.full[slot], bytes_row * (uint32_t)n);
      issue_stage(op, grp, r, n, koff, sm.ring[slot], &sm.full[slot], pol);
      ld_bytes += (uint64_t)bytes_row * n;
      ++pstage;
      if (pf_dist) prefetch_some();
    }
    if (!ok) break;
  }
  if (!ok || aborted(g)) {
    // Never leave the block with bulk copies in flight: wait (bounded) for the
    // most recent stages to land before returning.
    const uint32_t first = pstage > (uint32_t)NR ? pstage - NR : 0u;
    for (uint32_t s = first; s < pstage; ++s) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sm.full[s % NR], (s / NR) & 1u)) {
        if (globaltimer() - t0 > 200000000ull) break;
      }
    }
  }
}

// ------------------------------------------------------------------ consumer helpers
// The fp32 input vector h is stored permuted in shared memory so that the
// GEMV's loads are free of bank conflicts: lane l of a warp multiplies weight
// elements [8l + 256j, +8) and reads their inputs as two float4 at
// hperm(8l + 256j) and hperm(8l + 256j + 4), which for one j are 32
// consecutive float4.  hperm(k) for k a multiple of 4: element block m = k/8,
// half k/4 mod 2 -> ((m/32)*2 + half)*128 + 4*(m mod 32).
__device__ __forceinline__ int hperm(int k) {
  const int q = k >> 2, m = q >> 1;
  return (((m >> 5) << 1) + (q & 1)) * 128 + ((m & 31) << 2);
}

// Eight products of one 16-byte chunk of a bf16 row with the matching eight
// fp32 inputs, into two accumulators.
__device__ __forceinline__ void fma8(float (&acc)[2], const uint4 w, const float4 h0, const float4 h1) {
  acc[0] = fmaf(bf16_lo(w.x), h0.x, acc[0]);
  acc[1] = fmaf(bf16_hi(w.x), h0.y, acc[1]);
  acc[0] = fmaf(bf16_lo(w.y), h0.z, acc[0]);
  acc[1] = fmaf(bf16_hi(w.y), h0.w, acc[1]);
  acc[0] = fmaf(bf16_lo(w.z), h1.x, acc[0]);
  acc[1] = fmaf(bf16_hi(w.z), h1.y, acc[1]);
  acc[0] = fmaf(bf16_lo(w.w), h1.z, acc[0]);
  acc[1] = fmaf(bf16_hi(w.w), h1.w, acc[1]);
}

// Dot products of NR bf16 weight rows of a stage (and, with PAIR, of the NR
// partner rows `rps` rows further: gate and up) with the fp32 input vector h,
// all in shared memory.  One warp; lane l covers elements [8l + 256j, +8), so
// every 16-byte load of h serves all NR (or 2 NR) rows.  Row indices at or past
// `n` are clamped to the last row (their results are discarded).  Every lane
// returns every total.
template <int NR, bool PAIR>
__device__ __forceinline__ void dot_group(const uint8_t* stage, int i0, int n, int rps, const float* h, int K,
                                          int lane, float (&v)[NR], float (&u)[NR]) {
  const uint16_t* w[NR];
  const uint16_t* wu[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const int i = min(i0 + r, n - 1);
    w[r] = reinterpret_cast<const uint16_t*>(stage + (size_t)i * K * 2);
    wu[r] = reinterpret_cast<const uint16_t*>(stage + (size_t)(rps + i) * K * 2);
  }
  float a[NR][2], b[NR][2];
#pragma unroll
  for (int r = 0; r < NR; ++r) a[r][0] = a[r][1] = b[r][0] = b[r][1] = 0.f;
  const float* hp = h + lane * 4;  // hperm(8 lane + 256 j) = 256 j + 4 lane
#pragma unroll 2
  for (int e = lane * 8; e < K; e += 256, hp += 256) {
    const float4 h0 = *reinterpret_cast<const float4*>(hp);
    const float4 h1 = *reinterpret_cast<const float4*>(hp + 128);
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      fma8(a[r], *reinterpret_cast<const uint4*>(w[r] + e), h0, h1);
      if (PAIR) fma8(b[r], *reinterpret_cast<const uint4*>(wu[r] + e), h0, h1);
    }
  }
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    v[r] = warp_sum(a[r][0] + a[r][1]);
    u[r] = PAIR ? warp_sum(b[r][0] + b[r][1]) : 0.f;
  }
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

// Attention task modes: a chunk of the split-K ATTENTION operation (partials,
// merged by the last chunk to arrive), or a chunk of a fused
// projections+attention operation's kv-head group (tagged partials, merged by
// chunk 0).
constexpr int ATTN_SPLIT_OP = 0, ATTN_GROUP = 1;

__device__ __noinline__ bool attn_dispatch(Smem& sm, const Graph& g, const OpDesc& op, int j, int c, int C, int r,
                                           int mode, int cw, int lane, uint32_t iter, int worker);


// The LM head's last task to arrive (sm.last) turns every active column's
// maximum key into its next token: written to tokens[r, s+1] if that slot
// holds -1, always to pred; the request's step advances; the keys are reset.
// A prefill graph's columns are positions of one request: each column writes
// its own prediction, the last active one advances that request's step
// (every column reads the shared step before it changes).
__device__ __forceinline__ void argmax_tokens(Smem& sm, const Graph& g, const OpDesc& op, uint32_t iter, int ctid) {
  if (!sm.last) return;
  __threadfence();
  int s = 0, sn = 0, row = 0, qn = 0;
  bool act = false, next = false;
  unsigned long long key = 0ull;
  if (ctid < g.R) {
    act = request_state(g, ctid, iter, s, row);
    next = ctid + 1 < g.R && request_state(g, ctid + 1, iter, sn, qn);
    if (act) key = atomicAdd(op.keys + ctid, 0ull);
  }
  if (g.prefill) consumer_sync();
  if (ctid < g.R) {
    const int rq = ctid;
    if (act) {
      const int64_t nxt = (int64_t)argmax_key_index(key);
      int64_t* trow = g.tokens + (size_t)row * g.S;
      if (__ldcg(trow + s + 1) == -1) trow[s + 1] = nxt;
      if (op.pred != nullptr) op.pred[(size_t)row * g.S + s + 1] = nxt;
      if (!g.prefill || !next) g.step[row] = s + 1;
    }
    op.keys[rq] = 0ull;
  }
  consumer_sync();
  if (ctid == 0) red_release_add(g.events + (size_t)op.out_event * EVENT_STRIDE, 1u);
}

// ------------------------------------------------------------------ GEMV tasks
// Rows [row0,row1) of W (bf16, [rows, K] row-major) against one input vector h
// held in shared memory as fp32.  Each consumer warp owns whole rows (task
// row j goes to warp j % nwarps) and runs the operation's epilogue for them
// itself, so the weight stages need no block-wide barrier: every warp waits
// for each stage, computes its rows in it and releases the stage.
template <int KIND>
__device__ bool gemv_task(Smem& sm, const Graph& g, const OpDesc& op, int task, uint32_t iter,
                          uint32_t& cstage, int cw, int lane, int worker) {
  const int ctid = cw * 32 + lane;
  const int K = task_k(op), rps = op.rps, nw = op.nwarps;
  const bool split = KIND == TK_GEMV_RESID && op.ksplit > 1;
  const int koff = task_koff(op, task);
  int grp, row0, row1;
  task_rows(op, task, grp, row0, row1);
  float* hs = sm.u.g.hs;

  // ---- prologue: the input vector, fp32, in shared memory.  Every global
  // load of the prologue is issued before the first use (one L2 round trip).
  const int nrows = row1 - row0;
  const bool xs_ok = KIND == TK_GEMV_RESID && !split && nrows <= MAX_XS;
  // versions of the inputs (and of what this task writes)
  const uint32_t xtag = vtag(g, iter, op.x_writer) + op.tag_skew;
  const uint32_t atag = vtag(g, iter, op.a_writer) + op.tag_skew;
  const uint32_t mytag = vtag(g, iter, op.self);
  bool pfail = false;
  // consecutive claimed tasks of one dynamic op (same segment) share the
  // input vector already in shared memory
  const unsigned long long hkey =
      ((unsigned long long)iter << 32) | ((unsigned long long)op.self << 16) | (unsigned long long)task_seg(op, task);
  const bool reuse = op.dynamic && sm.h_key == hkey;
  if (KIND == TK_QKV_ATTN) {
    // What this operation's attention needs besides q, k and v, fetched while
    // the input is awaited: the request's position, its RoPE row, and the
    // ordering of the cache (this operation's attention releases its event
    // after appending; positions below s were appended in earlier iterations).
    if (ctid < op.d / 2) {
      int sp;
      const bool act = request_state(g, 0, iter, sp);
      if (act) sm.rope_row[ctid] = __ldg(op.rope + (size_t)sp * (op.d / 2) + ctid);
      if (ctid == 0) {
        sm.attn_s = act ? sp : -1;
        if (act && sp > 0) {
          // this task's share of the head's cached positions into L2, so the
          // group's attention (run by whichever task finishes last) reads
          // them at L2 latency
          const int tpg = op.ntasks / op.groups, t = task - grp * tpg;
          const int p0 = (int)(((long long)t * sp) / tpg), p1 = (int)(((long long)(t + 1) * sp) / tpg);
          if (p1 > p0) {
            const size_t base = (((size_t)op.layer * g.R) * op.Hkv + grp) * (size_t)op.S * op.d;
            const uint32_t bytes = (uint32_t)(p1 - p0) * (uint32_t)op.d * 2u;
            prefetch_l2(op.kc + base + (size_t)p0 * op.d, bytes);
            prefetch_l2(op.vc + base + (size_t)p0 * op.d, bytes);
          }
        }
      }
    }
    if (ctid == 0 && iter > 0 &&
        !wait_counter(g, g.events + (size_t)op.out_event * EVENT_STRIDE, iter * (uint32_t)op.out_trigger, 1, op.self,
                      task, worker, (int)iter))
      pfail = true;
  }
  if (KIND == TK_GEMV_RESID) {
    // the input (this task's segment of it) into shared memory once every
    // element carries its writer's tag, the task's residual rows likewise;
    // all loads are issued before any tag is looked at
    constexpr int NC = MAX_K / (CONSUMER_THREADS * 4);
    constexpr int NX = MAX_XS / CONSUMER_THREADS;
    uint64_t aw[NC * 4], xw[NX];
    const bool load_a = !reuse;
    auto a_addr = [&](int u) { return op.a_in + koff + ((u / 4) * CONSUMER_THREADS + ctid) * 4 + (u % 4); };
    auto a_valid = [&](int u) { return load_a && ((u / 4) * CONSUMER_THREADS + ctid) * 4 < K; };
    auto x_addr = [&](int q) { return op.x_out + row0 + q * CONSUMER_THREADS + ctid; };
    auto x_valid = [&](int q) { return xs_ok && q * CONSUMER_THREADS + ctid < nrows; };
#pragma unroll
    for (int c = 0; c < NC; ++c)
      if (a_valid(4 * c)) {
        ld_tagged2(a_addr(4 * c), aw[4 * c], aw[4 * c + 1]);
        ld_tagged2(a_addr(4 * c + 2), aw[4 * c + 2], aw[4 * c + 3]);
      }
#pragma unroll
    for (int q = 0; q < NX; ++q)
      if (x_valid(q)) xw[q] = ld_tagged(x_addr(q));
    pfail |= !settle_tagged(g, aw, a_addr, a_valid, atag, op.self, worker, (int)iter);
    pfail |= !settle_tagged(g, xw, x_addr, x_valid, xtag, op.self, worker, (int)iter);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int k = (c * CONSUMER_THREADS + ctid) * 4;
      if (a_valid(4 * c))
        *reinterpret_cast<float4*>(hs + hperm(k)) = make_float4(word_value(aw[4 * c]), word_value(aw[4 * c + 1]),
                                                                word_value(aw[4 * c + 2]), word_value(aw[4 * c + 3]));
    }
#pragma unroll
    for (int q = 0; q < NX; ++q)
      if (x_valid(q)) sm.u.g.xs[q * CONSUMER_THREADS + ctid] = word_value(xw[q]);
  } else if (!reuse) {
    // RMSNorm: x and the norm weight are read once into registers, the
    // statistics are reduced in a fixed order.
    constexpr int NCH = MAX_NORM_K / (CONSUMER_THREADS * 8);
    float xr[NCH][8];
    uint4 wr[NCH];
    uint64_t xw[NCH * 8];
    auto x_addr = [&](int u) { return op.x + ((u / 8) * CONSUMER_THREADS + ctid) * 8 + (u % 8); };
    auto x_valid = [&](int u) { return ((u / 8) * CONSUMER_THREADS + ctid) * 8 < K; };
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int k = (c * CONSUMER_THREADS + ctid) * 8;
      if (k < K) wr[c] = __ldg(reinterpret_cast<const uint4*>(op.norm_w + k));
    }
    // all of the task's x words issued before any is looked at
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        if (x_valid(8 * c)) ld_tagged2(x_addr(8 * c + e), xw[8 * c + e], xw[8 * c + e + 1]);
        else xw[8 * c + e] = xw[8 * c + e + 1] = 0ull;
      }
    }
    pfail |= !settle_tagged(g, xw, x_addr, x_valid, xtag, op.self, worker, (int)iter);
#pragma unroll
    for (int c = 0; c < NCH; ++c)
#pragma unroll
      for (int e = 0; e < 8; ++e) xr[c][e] = word_value(xw[8 * c + e]);
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int k = (c * CONSUMER_THREADS + ctid) * 8;
      if (k < K) {
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(xr[c][e], xr[c][e], ss);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) sm.ss[cw] = ss;
    consumer_sync();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < CONSUMER_WARPS; ++w) tot += sm.ss[w];
    const float rinv = 1.0f / sqrtf(tot / (float)K + op.eps);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int k = (c * CONSUMER_THREADS + ctid) * 8;
      if (k < K) {
        const uint4 w = wr[c];
        float4 h0, h1;
        h0.x = xr[c][0] * rinv * bf16_lo(w.x); h0.y = xr[c][1] * rinv * bf16_hi(w.x);
        h0.z = xr[c][2] * rinv * bf16_lo(w.y); h0.w = xr[c][3] * rinv * bf16_hi(w.y);
        h1.x = xr[c][4] * rinv * bf16_lo(w.z); h1.y = xr[c][5] * rinv * bf16_hi(w.z);
        h1.z = xr[c][6] * rinv * bf16_lo(w.w); h1.w = xr[c][7] * rinv * bf16_hi(w.w);
        *reinterpret_cast<float4*>(hs + hperm(k)) = h0;
        *reinterpret_cast<float4*>(hs + hperm(k + 4)) = h1;
      }
    }
  }
  if (consumer_sync_or(pfail)) return false;
  if (ctid == 0) sm.h_key = hkey;  // every thread read the previous key before the barrier
  if (g.profiling && ctid == 0) sm.t_pro = globaltimer();

  const bool capture = (g.capture_iter == (int)iter);
  unsigned long long best = 0ull;
  bool fail = false;

  // Epilogue of task-local row j with its full dot product(s).
  auto finish = [&](int j, float v, float u) {
    const int row = row0 + j;
    if (KIND == TK_NORM_GEMV || KIND == TK_QKV_ATTN) {
      const int sg = seg_of(op, row);
      st_tagged(op.y[sg] + seg_row(op, grp, sg, row), v, mytag);
    } else if (KIND == TK_GEMV_RESID) {
      if (split) {
        st_tagged(op.kpart + (size_t)task_seg(op, task) * op.N + row, v, mytag);
        return;
      }
      float xo;
      if (xs_ok) xo = sm.u.g.xs[j];
      else poll_tagged(g, op.x_out + row, ld_tagged(op.x_out + row), xtag, xo, op.self, worker, (int)iter);
      const float nx = xo + v;
      st_tagged(op.x_out + row, nx, mytag);
      if (capture && op.capture_slot >= 0 && g.cap_hidden != nullptr)
        g.cap_hidden[(size_t)op.capture_slot * g.R * g.H + row] = nx;
    } else if (KIND == TK_NORM_GEMV_SILU) {
      st_tagged(op.a_out + row, silu_f(v) * u, mytag);
    } else {  // LM head
      const unsigned long long key = argmax_key(v, (uint32_t)row);
      best = key > best ? key : best;
      if (capture && g.cap_logits != nullptr) g.cap_logits[row] = v;
    }
  };


  // Each warp owns groups of RB whole rows that share every load of h from
  // shared memory (gate/up: one gate row and one up row); group u of the task
  // goes to warp u % nwarps.  RB = 2 measured best for single matrices: it
  // halves the shared-memory reads of h, more rows per warp leave too few
  // warps working on each stage.
  constexpr bool PAIR = KIND == TK_NORM_GEMV_SILU;
  constexpr int RB = PAIR ? 1 : 2;
  int un = cw;     // next task-local group of this warp
  int ubase = 0;   // first group of the current stage
  for (int base = 0; base < nrows; base += rps) {
    const int n = min(rps, nrows - base);
    const int ngroups = (n + RB - 1) / RB;
    const uint32_t slot = cstage % NSTAGES;
    bool ok = true;
    if (lane == 0) {
      const uint64_t w0 = (g.profiling && ctid == 0) ? globaltimer() : 0ull;
      ok = wait_mbar(g, &sm.full[slot], (cstage / NSTAGES) & 1u, 3, worker);
      if (g.profiling && ctid == 0) {
        const uint64_t w1 = globaltimer();
        sm.t_stall += w1 - w0;
        sm.t_last = w1;
        if (base == 0) sm.t_data = w1;
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
    if (!ok) {
      fail = true;
      break;
    }
    const uint8_t* stage = sm.ring[slot];
    if (cw < nw) {
      for (; un < ubase + ngroups; un += nw) {
        const int i0 = (un - ubase) * RB;
        float v[RB], u[RB];
        dot_group<RB, PAIR>(stage, i0, n, rps, hs, K, lane, v, u);
#pragma unroll
        for (int r = 0; r < RB; ++r)
          if (lane == r && i0 + r < n) finish(base + i0 + r, v[r], u[r]);
      }
    }
    ubase += ngroups;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[slot]);
    ++cstage;
  }
  if (KIND == TK_NORM_GEMV_ARGMAX) best = warp_max_u64(best);
  if (KIND == TK_NORM_GEMV_ARGMAX && lane == 0) sm.bestk[cw] = best;
  if (consumer_sync_or(fail)) return false;
  if (g.profiling && ctid == 0) sm.t_loop = globaltimer();

  if (split) {
    // The last segment task of this row block to finish adds the partial sums
    // to the residual, in segment order.
    // (no fence: the finisher waits for the partials' tags)
    if (ctid == 0) {
      const uint32_t old = atomicAdd(op.blk_cnt + task % (op.ntasks / op.ksplit), 1u);
      sm.last = ((old + 1u) % (uint32_t)op.ksplit) == 0u;
    }
    consumer_sync();
    if (sm.last) {
      bool ffail = false;
      for (int j = ctid; j < nrows; j += CONSUMER_THREADS) {
        const int row = row0 + j;
        // every partial and the residual loaded before any tag is looked at
        constexpr int MAXS = MAX_KSPLIT;
        uint64_t pw[MAXS], xw[1];
        auto p_addr = [&](int k) { return op.kpart + (size_t)k * op.N + row; };
        auto p_valid = [&](int k) { return k < op.ksplit; };
        auto x_addr = [&](int) { return op.x_out + row; };
        auto x_valid = [](int) { return true; };
#pragma unroll
        for (int k = 0; k < MAXS; ++k)
          if (p_valid(k)) pw[k] = ld_tagged(p_addr(k));
        xw[0] = ld_tagged(x_addr(0));
        ffail |= !settle_tagged(g, pw, p_addr, p_valid, mytag, op.self, worker, (int)iter);
        ffail |= !settle_tagged(g, xw, x_addr, x_valid, xtag, op.self, worker, (int)iter);
        float sum = 0.f;
#pragma unroll
        for (int k = 0; k < MAXS; ++k)
          if (p_valid(k)) sum = k == 0 ? word_value(pw[k]) : sum + word_value(pw[k]);
        const float xo = word_value(xw[0]);
        const float nx = xo + sum;
        st_tagged(op.x_out + row, nx, mytag);
        if (capture && op.capture_slot >= 0 && g.cap_hidden != nullptr)
          g.cap_hidden[(size_t)op.capture_slot * g.R * g.H + row] = nx;
      }
      if (consumer_sync_or(ffail)) return false;
    }
  }

  if (KIND == TK_QKV_ATTN && op.group_sync) {
    // The group's first op.C tasks each attend to a chunk of the positions
    // (once the group's q, k, v carry their tags) and chunk 0 merges; each
    // task of the operation runs on its own worker, so the waits on the
    // group's other tasks always end.
    const int tpg = op.ntasks / op.groups, t = task - grp * tpg;
    if (t < op.C && !attn_dispatch(sm, g, op, grp, t, op.C, 0, ATTN_GROUP, cw, lane, iter, worker)) return false;
    if (t == 0) {
      consumer_sync();
      if (ctid == 0) red_release_add(g.events + (size_t)op.out_event * EVENT_STRIDE, 1u);
    }
  } else if (KIND == TK_QKV_ATTN) {
    // More tasks than workers: the last projection task of this kv head's
    // group to finish runs the group's attention.  (No fence: the attention
    // waits for q, k and v through their tags.)
    if (ctid == 0) {
      const uint32_t old = atomicAdd(op.grp_cnt + grp, 1u);
      sm.last = ((old + 1u) % (uint32_t)(op.ntasks / op.groups)) == 0u;
    }
    consumer_sync();
    if (sm.last) {
      // the same chunks as in group mode, one after another, chunk 0 (the
      // merge) last: results are identical whichever mode runs
      for (int cc = op.C - 1; cc >= 0; --cc)
        if (!attn_dispatch(sm, g, op, grp, cc, op.C, 0, ATTN_GROUP, cw, lane, iter, worker)) return false;
      consumer_sync();
      if (ctid == 0) red_release_add(g.events + (size_t)op.out_event * EVENT_STRIDE, 1u);
    }
  }

  if (KIND == TK_NORM_GEMV_ARGMAX) {
    // Per-task maximum -> one 64-bit atomicMax; the last task to arrive
    // finishes the iteration.
    if (ctid == 0) {
      unsigned long long b = 0ull;
      for (int w = 0; w < CONSUMER_WARPS; ++w) b = sm.bestk[w] > b ? sm.bestk[w] : b;
      atomicMax(op.keys, b);
      __threadfence();
      const uint32_t old = atomicAdd(op.arrive, 1u);
      sm.last = ((old + 1u) % (uint32_t)op.ntasks) == 0u;
    }
    consumer_sync();
    argmax_tokens(sm, g, op, iter, ctid);
  }
  return true;
}

// ------------------------------------------------------------------ batched projections (tensor cores)
#include "mpk_batch.cuh"

template <int BW>
__device__ __forceinline__ void bgemm_advance(const OpDesc& op, int task, uint32_t& cstage, uint32_t& accn) {
  uint32_t st, bl;
  bgemm_counts<BW>(op, task, st, bl);
  cstage += st;
  accn += bl;
}

// ------------------------------------------------------------------ attention on the tensor cores
// The split-K operation's main loop: the chunk's cached positions arrive
// through the ring (stages of PB positions, K then V, 128-byte swizzled boxes
// of 64 dims), the positions the iteration itself produced are rows KX / VX in
// shared memory (row a0r + t, nin of them).  Warp-level MMAs (m16n8k16, bf16
// inputs, fp32 accumulation), one 16-position tile per warp and stage; warp w
// takes tile w % T16 and dims d0 = 64 (w / T16) .. d0 + 63 (d = 128: the
// tile's two warps split the head dim):
//  * scores S = Q K^T (16 x 16): A = the queries, rows 0..3 the bf16 part
//    hi(q) of query heads 0..3, rows 4..7 the rest lo(q) = bf16(q - hi(q)),
//    rows 8..15 zero; B = the tile's k rows.  Score of head h = row h + row
//    h + 4 (lanes 16 apart): the products of the fp32 queries to ~16 bits.
//    With d = 128 each warp of the tile sums over its own 64 dims and the
//    two add their halves through shared memory behind a two-warp barrier;
//  * online softmax in base 2 per head over the tile (the queries carry
//    log2(e) / sqrt(d)), positions past the valid count masked;
//  * O^T += V^T P^T (16 dims x 8 columns per MMA): A = the tile's v rows
//    loaded transposed (zeroed past the valid count, where the rows may hold
//    anything), B = the probabilities straight from the score fragments,
//    column h the hi part and column h + 4 the lo part of head h.
// The warp's (max, sum, output) go to A.wm / A.wacc for the block merge.
template <int G, int D>
__device__ __forceinline__ bool attn_stream_mma(Smem& sm, const Graph& g, const OpDesc& op, AttnScratch& A, int lo,
                                                int chi, int a0r,
                                                int nin, const uint16_t* KX, const uint16_t* VX, int cw, int lane,
                                                int worker, uint32_t& cstage) {
  constexpr int PB = STAGE_BYTES / (4 * D);  // positions per stage
  constexpr int T16 = PB / 16;               // tiles per stage
  constexpr int KS = D / 16;                 // k-steps of the scores
  static_assert(G <= 4 && (CONSUMER_WARPS / T16) * 64 == D && T16 * (CONSUMER_WARPS / T16) == CONSUMER_WARPS,
                "one tile and 64 dims of v per warp");
  const int tile = cw % T16, d0 = (cw / T16) * 64;
  const int gq = lane >> 2, tq = lane & 3, hq = gq & 3;
  const bool lo_row = gq >= 4;
  const uint32_t full_mask = 0xffffffffu;
  // bf16 hi / lo part of x for this lane's row of the query / probability operand
  auto part = [&](float x) -> uint32_t {
    const uint16_t h = f32_to_bf16_rn(x);
    return lo_row ? (uint32_t)f32_to_bf16_rn(x - __uint_as_float((uint32_t)h << 16)) : (uint32_t)h;
  };
  // with two warps per tile (d = 128) each computes the scores over its own
  // 64 dims and the pair adds the halves through shared memory
  constexpr bool PAIR = T16 * 2 == CONSUMER_WARPS;
  constexpr int KSW = PAIR ? KS / 2 : KS;  // k-steps this warp takes
  const int kd0 = PAIR ? d0 : 0;
  uint32_t qa[KSW][2];
#pragma unroll
  for (int ks = 0; ks < KSW; ++ks) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int d = kd0 + 16 * ks + 8 * hf + 2 * tq;
      const float x0 = hq < G ? A.qs[hq * D + d] : 0.f;
      const float x1 = hq < G ? A.qs[hq * D + d + 1] : 0.f;
      qa[ks][hf] = part(x0) | (part(x1) << 16);
    }
  }
  // O^T fragments: dims d0 + 16 mt + gq (elements 0, 1) and + 8 (2, 3), columns 2 tq, 2 tq + 1
  float o[4][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;
  float m = -INFINITY, l = 0.f;  // head hq's running max and this lane's share of its sum
  const int src_a = 4 * ((2 * tq) & 3), src_b = 4 * ((2 * tq + 1) & 3);  // lanes holding the columns' heads

  // The current tile: K rows at kb, V rows at vb, either a ring stage
  // (swizzled boxes) or, for the iteration's own rows, plain [row][d] rows
  // a0r.. (own > 0 of them; rows past them read the last, then masked).
  // addr(base, t, c) = shared address of dims 8c..8c+7 of the tile's row t.
  uint32_t kb = 0, vb = 0;
  int own = 0;
  auto addr = [&](uint32_t base, int t, int c) -> uint32_t {
    if (own == 0)  // box c / 8, 128-byte row t, 16-byte unit c % 8 swizzled by the row
      return base + (uint32_t)(c >> 3) * (uint32_t)(PB * 128) + (uint32_t)t * 128u +
             (uint32_t)(((c & 7) ^ (t & 7)) << 4);
    return base + (uint32_t)((a0r + min(t, own - 1)) * D * 2 + c * 16);
  };
  // one tile of nv valid rows (1..16)
  auto run_tile = [&](int nv) {
    // two accumulators per 8 positions (even / odd k-steps): shorter MMA chains
    float sa[2][2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) sa[nt][h][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSW / 2; ++kk) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(addr(kb, nt * 8 + (lane & 7), kd0 / 8 + 4 * kk + (lane >> 3)), b0, b1, b2, b3);
        mma_bf16_16816(sa[nt][0], qa[2 * kk][0], 0u, qa[2 * kk][1], 0u, b0, b1);
        mma_bf16_16816(sa[nt][1], qa[2 * kk + 1][0], 0u, qa[2 * kk + 1][1], 0u, b2, b3);
      }
    }
    if (PAIR) {
      float4* xs = A.xs;  // [warp][lane] partial scores (rows g)
      xs[cw * 32 + lane] = make_float4(sa[0][0][0] + sa[0][1][0], sa[0][0][1] + sa[0][1][1],
                                       sa[1][0][0] + sa[1][1][0], sa[1][0][1] + sa[1][1][1]);
      named_sync(3 + tile, 64);  // the tile's two warps (barriers 0..2 serve the block and the epilogue)
      const float4 ps = xs[(cw ^ T16) * 32 + lane];
      sa[0][1][0] += ps.x;
      sa[0][1][1] += ps.y;
      sa[1][1][0] += ps.z;
      sa[1][1][1] += ps.w;
    }
    // this lane's positions: 2 tq, 2 tq + 1 (nt = 0) and 8 + 2 tq, 9 + 2 tq (nt = 1)
    float sc[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float x = sa[nt][0][e] + sa[nt][1][e];
        const float v = x + __shfl_xor_sync(full_mask, x, 16);
        sc[nt * 2 + e] = (nt * 8 + 2 * tq + e < nv) ? v : -INFINITY;
      }
    float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mx = fmaxf(mx, __shfl_xor_sync(full_mask, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(full_mask, mx, 2));
    const float mn = fmaxf(m, mx);   // finite: position 0 of the tile is valid
    const float al = exp2f(m - mn);  // m = -inf -> 0
    float p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = exp2f(sc[i] - mn);  // masked -> 0
    l = fmaf(l, al, (p[0] + p[1]) + (p[2] + p[3]));
    m = mn;
    const float al_a = __shfl_sync(full_mask, al, src_a), al_b = __shfl_sync(full_mask, al, src_b);
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      o[mt][0] *= al_a;
      o[mt][1] *= al_b;
      o[mt][2] *= al_a;
      o[mt][3] *= al_b;
    }
    const uint32_t pb0 = part(p[0]) | (part(p[1]) << 16);
    const uint32_t pb1 = part(p[2]) | (part(p[3]) << 16);
    const bool ragged = nv < 16;
    auto keep = [&](uint32_t v, int t) -> uint32_t {
      return (t < nv ? (v & 0xffffu) : 0u) | (t + 1 < nv ? (v & 0xffff0000u) : 0u);
    };
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      // matrices: rows 0..7 / 8..15 of the tile (lanes 16..31 the second) x
      // 8 dims at chunk c / c + 1 (lanes 8..15 and 24..31 the second)
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(addr(vb, (lane & 7) + ((lane >> 4) << 3), d0 / 8 + 2 * mt + ((lane >> 3) & 1)), a0, a1, a2, a3);
      if (ragged) {
        a0 = keep(a0, 2 * tq);
        a1 = keep(a1, 2 * tq);
        a2 = keep(a2, 8 + 2 * tq);
        a3 = keep(a3, 8 + 2 * tq);
      }
      mma_bf16_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
    }
  };

  // Stages: one elected thread waits (bounded), the block learns the outcome
  // through the barrier; once every warp is done with its tile the stage is
  // released (one arrival per consumer warp on the GEMV ring, one on the
  // tensor-core ring).  Measured faster than per-warp waits and releases.
  const bool elected = cw == 0 && lane == 0;
  const int nr = g.batched ? NSTB : NSTAGES;
  auto release = [&](uint32_t sl) {
    const int arrivals = g.batched ? 1 : CONSUMER_WARPS;
    for (int a = 0; a < arrivals; ++a) mbar_arrive(&sm.empty[sl]);
  };
  uint32_t prev = 0;
  bool sfail = false;
  for (int p0 = lo; p0 < chi; p0 = attn_stage_end(op, p0, chi, PB)) {
    const int n = attn_stage_end(op, p0, chi, PB) - p0;
    const uint32_t cs = cstage;
    const uint32_t slot = cs % (uint32_t)nr;
    bool okk = true;
    if (elected) okk = wait_mbar(g, &sm.full[slot], (cs / (uint32_t)nr) & 1u, 3, worker);
    if (consumer_sync_or(!okk)) {
      sfail = true;
      break;
    }
    // every warp is past the previous stage: release it
    if (elected && p0 > lo) release(prev);
    const int nv = min(16, n - tile * 16);
    if (nv > 0) {
      kb = smem_u32(sm.ring[slot]) + (uint32_t)(tile * 16) * 128u;  // tiles start on 1024-byte boundaries
      vb = kb + (uint32_t)(STAGE_BYTES / 2);
      run_tile(nv);
    }
    prev = slot;
    cstage = cs + 1u;
  }
  if (consumer_sync_or(sfail)) return false;
  if (elected && chi > lo) release(prev);
  if (tile == 0 && nin > 0) {
    // the iteration's own rows
    own = nin;
    kb = smem_u32(KX);
    vb = smem_u32(VX);
    run_tile(nin);
  }
  // the warp's partial: the head's sum over the lanes of its row, the output
  // as hi column + lo column (lanes 2 apart)
  l += __shfl_xor_sync(full_mask, l, 1);
  l += __shfl_xor_sync(full_mask, l, 2);
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float ov = o[mt][e] + __shfl_xor_sync(full_mask, o[mt][e], 2);
      const int h = 2 * tq + (e & 1), d = d0 + 16 * mt + gq + 8 * (e >> 1);
      if (tq < 2 && h < G) A.wacc[cw][h * D + d] = ov;
    }
  }
  if (!lo_row && hq < G && tq == 0) {
    A.wm[cw][hq][0] = m;
    A.wm[cw][hq][1] = l;
  }
  return true;
}

// ------------------------------------------------------------------ attention task
// Attention of kv head j for request r at position s, over the positions
// [c (s+1) / C, (c+1) (s+1) / C) of chunk c of C.  Prologue: RMSNorm over the
// head dim and rotate-half RoPE of the G query heads of the group and of k;
// the cache append of k, v at s (by the chunk holding s, or in group mode by
// chunk 0).  Main loop: LP = D/8 lanes per position (8 dims per lane), 32/LP
// positions per warp step, NSTEP steps' K/V loads issued before any is used,
// online softmax in base 2 per query head.  The chunk's (max, sum,
// unnormalised output) partial goes to global memory; the split operation's
// last chunk task of (r, j) to arrive merges the partials in chunk order and
// signals the operation's event, in group mode chunk 0 merges once every
// partial carries this iteration's tag and writes o.
template <int G, int D, bool STREAMED>
__device__ __forceinline__ bool attn_task(Smem& sm, const Graph& g, const OpDesc& op, int j, int c, int C, int r,
                                          int mode, int cw, int lane, uint32_t iter, int worker, uint32_t cstage) {
  // the fused operation (group mode, state fetched in the projections'
  // prologue) reads the cache itself; the split-K operation streams it.  A
  // run-time flag, although it follows STREAMED: measured, the compile-time
  // form makes the fused operation's register allocation slower
  const bool fused = mode == ATTN_GROUP;
  if (cw == 0 && lane == 0) sm.h_key = ~0ull;  // the attention scratch overlays the GEMV input vector
  constexpr int LP = D / 8;          // lanes per position
  constexpr int PPW = 32 / LP;       // positions per warp step
  constexpr int NSTEP = 4;           // warp steps whose loads are in flight together
  constexpr float LOG2E = 1.4426950408889634f;
  const int ctid = cw * 32 + lane;
  const int Hkv = op.Hkv;
  AttnScratch& A = sm.u.a;
  // the fused operation's cache rows (one request, contiguous cache)
  size_t kvbase = ((((size_t)op.layer * g.Rq + r) * Hkv + j) * (size_t)op.S) * D;
  // k and v (bf16, k normalised and rotated) of the positions the iteration
  // itself produces: row 0 the task's own position (A.ks, A.vs); prefill: row
  // c the position of column c of the chunk, in the ring stage that the
  // tensor-core path keeps for its input rows (free while an attention task
  // runs: every MMA of the previous projection task has completed)
  const bool pf = g.prefill;  // prefill graphs run split-K attention only
  const int own = pf ? r : 0;
  uint16_t* const KX = pf ? reinterpret_cast<uint16_t*>(sm.ring[NSTB]) : A.ks;
  uint16_t* const VX = pf ? reinterpret_cast<uint16_t*>(sm.ring[NSTB]) + MAX_PREFILL * MAX_D : A.vs;
  const int CS = op.C;  // split op: chunk partials per (request, query head)
  const float* pbase = op.part + (((size_t)r * op.Hq + (size_t)j * G) * CS) * (D + 2);
  // Prologue rows: warp cw < G takes query head cw of the group, warp G the
  // key, warp G+1 the value.  Their loads do not depend on the step, so they
  // are issued before it is read.
  constexpr int EL = D / 32;  // elements per lane
  const int prow = cw;
  const uint32_t intag = vtag(g, iter, op.a_writer) + op.tag_skew;
  const uint32_t mytag = vtag(g, iter, op.self);
  float x[EL];
  uint64_t xw[EL];
  const uint64_t* src = prow < G ? op.q + (size_t)r * op.Hq * D + (size_t)(j * G + prow) * D
                      : prow == G ? op.k + (size_t)r * Hkv * D + (size_t)j * D
                                  : op.v + (size_t)r * Hkv * D + (size_t)j * D;
  if (prow < G + 2) {
#pragma unroll
    for (int e = 0; e < EL; ++e) xw[e] = ld_tagged(src + lane + 32 * e);
  }
  int s;
  bool active;
  bool afail = false;
  size_t sdst = 0;  // element offset of position s in the caches (the append)
  if (fused) {
    // fused with the projections: state fetched in that task's prologue
    s = sm.attn_s;
    active = s >= 0;
  } else {
    int q;
    active = request_state(g, r, iter, s, q);
    if constexpr (STREAMED) {
      if (active) {
        const int row = kv_row(g, op, q, j, s);
        if (row < 0) {
          if (ctid == 0) record_error(g, -11 /*DEVICE*/, 12, op.self, -1, worker, (int)iter, (uint32_t)q, (uint32_t)s);
          afail = true;
        } else {
          sdst = (size_t)row * D;
        }
      }
    } else {
      kvbase = ((((size_t)op.layer * g.Rq + q) * Hkv + j) * (size_t)op.S) * D;
    }
  }
  if (active && prow < G + 2) {
    // q, k, v of this iteration (their tags), then the cache: positions below
    // s were appended by this operation's attention tasks of earlier
    // iterations, which released its event after appending
#pragma unroll
    for (int e = 0; e < EL; ++e) {
      if (word_tag(xw[e]) == intag) x[e] = word_value(xw[e]);
      else afail |= !poll_tagged(g, src + lane + 32 * e, xw[e], intag, x[e], op.self, worker, (int)iter);
    }
  }
  if (!fused && active && ctid == 0 && iter > 0 &&
      !wait_counter(g, g.events + (size_t)op.out_event * EVENT_STRIDE, iter * (uint32_t)op.out_trigger, 1, op.self,
                    -1, worker, (int)iter))
    afail = true;

  if (active) {
    const int npos = s + 1;
    int lo, hi;
    if constexpr (STREAMED) {
      chunk_bounds(op, c, C, npos, lo, hi);
    } else {
      lo = (int)(((long long)c * npos) / C);
      hi = (int)(((long long)(c + 1) * npos) / C);
    }
    if (prow < G + 2) {
      if (prow <= G) {
        float2 rc[EL / 2];
        const float2* cs = op.rope + (size_t)s * (D / 2);
#pragma unroll
        for (int e = 0; e < EL / 2; ++e) rc[e] = fused ? sm.rope_row[lane + 32 * e] : __ldg(cs + lane + 32 * e);
        const uint16_t* wn = prow < G ? op.qn_w : op.kn_w;
        uint16_t wb[EL];
#pragma unroll
        for (int e = 0; e < EL; ++e) wb[e] = __ldg(wn + lane + 32 * e);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < EL; ++e) ss = fmaf(x[e], x[e], ss);
        ss = warp_sum(ss);
        const float rinv = 1.0f / sqrtf(ss / (float)D + op.eps);
#pragma unroll
        for (int e = 0; e < EL; ++e) x[e] = x[e] * rinv * __uint_as_float((uint32_t)wb[e] << 16);
        // rotate-half RoPE: element i pairs with i + D/2 (same lane, e + EL/2)
#pragma unroll
        for (int e = 0; e < EL / 2; ++e) {
          const float2 t = rc[e];
          const float a = x[e], b = x[e + EL / 2];
          x[e] = a * t.x - b * t.y;
          x[e + EL / 2] = b * t.x + a * t.y;
        }
      }
#pragma unroll
      for (int e = 0; e < EL; ++e) {
        const int i = lane + 32 * e;
        if (prow < G) A.qs[prow * D + i] = x[e] * (LOG2E / sqrtf((float)D));
        else if (prow == G) KX[own * D + i] = f32_to_bf16_rn(x[e]);
        else VX[own * D + i] = f32_to_bf16_rn(x[e]);
      }
    }
    if (pf) {
      // the chunk's earlier positions this task attends to (columns below
      // r, produced in this iteration and not read from the cache): their k
      // (normalised, rotated at its own position) and v, one row per warp
      const int sc0 = chunk0(g, r, s), a0 = lo > sc0 ? lo : sc0, b0 = hi < s ? hi : s;
      for (int row = cw; row < 2 * (b0 - a0); row += CONSUMER_WARPS) {
        const int pos = a0 + row / 2, rp = pos - sc0;
        const bool isk = (row & 1) == 0;
        const uint64_t* rs = (isk ? op.k : op.v) + (size_t)rp * Hkv * D + (size_t)j * D;
        float y[EL];
#pragma unroll
        for (int e = 0; e < EL; ++e) {
          const uint64_t w = ld_tagged(rs + lane + 32 * e);
          if (word_tag(w) == intag) y[e] = word_value(w);
          else afail |= !poll_tagged(g, rs + lane + 32 * e, w, intag, y[e], op.self, worker, (int)iter);
        }
        if (isk) {
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < EL; ++e) ss = fmaf(y[e], y[e], ss);
          ss = warp_sum(ss);
          const float rinv = 1.0f / sqrtf(ss / (float)D + op.eps);
#pragma unroll
          for (int e = 0; e < EL; ++e)
            y[e] = y[e] * rinv * __uint_as_float((uint32_t)__ldg(op.kn_w + lane + 32 * e) << 16);
          const float2* cs = op.rope + (size_t)pos * (D / 2);
#pragma unroll
          for (int e = 0; e < EL / 2; ++e) {
            const float2 t = __ldg(cs + lane + 32 * e);
            const float a = y[e], b = y[e + EL / 2];
            y[e] = a * t.x - b * t.y;
            y[e + EL / 2] = b * t.x + a * t.y;
          }
        }
#pragma unroll
        for (int e = 0; e < EL; ++e) (isk ? KX : VX)[rp * D + lane + 32 * e] = f32_to_bf16_rn(y[e]);
      }
    }
    // the rows sit in memory the tensor cores' bulk copies rewrite later
    if (pf) fence_proxy_async_smem();
    if (consumer_sync_or(afail)) return false;
    // the cache append at s: by the chunk holding s, or in group mode by the
    // merging task (chunk 0), whose release after the merge covers it
    if ((mode == ATTN_GROUP ? c == 0 : hi == npos) && ctid < D / 4) {
      // append k (first D/8 threads) and v (next D/8) at position s: 16 B each
      const int half = D / 8;
      const int which = ctid / half, q8 = ctid % half;
      uint16_t* dst;
      if constexpr (STREAMED) dst = (which == 0 ? op.kc : op.vc) + sdst + q8 * 8;
      else dst = (which == 0 ? op.kc : op.vc) + kvbase + (size_t)s * D + q8 * 8;
      const uint16_t* srcs = (which == 0 ? KX : VX) + own * D + q8 * 8;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(srcs);
    }

    // ---- main loop
    if constexpr (STREAMED) {
      // Split-K operation: the chunk's cached positions [lo, min(hi, chunk
      // start)) arrive through the weight ring and run on the tensor cores;
      // the positions this iteration produced (s, and prefill: the chunk's
      // earlier columns) come from their rows in shared memory
      const int sc0 = chunk0(g, r, s);
      const int chi = hi < sc0 ? hi : sc0;
      const int a0 = lo > sc0 ? lo : sc0;
      if (!attn_stream_mma<G, D>(sm, g, op, A, lo, chi, a0 - sc0, hi - a0, KX, VX, cw, lane, worker, cstage))
        return false;
    } else {
      // fused operation: the positions straight from the cache (and s from
      // shared memory), LP lanes per position on the CUDA cores
      const int grp = lane / LP, sub = lane % LP;
      float acc[G][8], m[G], l[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        m[hh] = -INFINITY;
        l[hh] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[hh][e] = 0.f;
      }
      // one position's K/V (8 dims per lane) into the warp's online softmax
      auto consume = [&](const uint4 kvu, const uint4 vvu, bool valid) {
        const float kf[8] = {bf16_lo(kvu.x), bf16_hi(kvu.x), bf16_lo(kvu.y), bf16_hi(kvu.y),
                             bf16_lo(kvu.z), bf16_hi(kvu.z), bf16_lo(kvu.w), bf16_hi(kvu.w)};
        float sc[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float4 q0 = *reinterpret_cast<const float4*>(A.qs + hh * D + sub * 8);
          const float4 q1 = *reinterpret_cast<const float4*>(A.qs + hh * D + sub * 8 + 4);
          float a = q0.x * kf[0];
          a = fmaf(q0.y, kf[1], a); a = fmaf(q0.z, kf[2], a); a = fmaf(q0.w, kf[3], a);
          a = fmaf(q1.x, kf[4], a); a = fmaf(q1.y, kf[5], a); a = fmaf(q1.z, kf[6], a); a = fmaf(q1.w, kf[7], a);
#pragma unroll
          for (int o = 1; o < LP; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
          sc[hh] = a;
        }
        if (valid) {
          const float vf[8] = {bf16_lo(vvu.x), bf16_hi(vvu.x), bf16_lo(vvu.y), bf16_hi(vvu.y),
                               bf16_lo(vvu.z), bf16_hi(vvu.z), bf16_lo(vvu.w), bf16_hi(vvu.w)};
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            const float mn = fmaxf(m[hh], sc[hh]);
            const float al = exp2f(m[hh] - mn);  // m = -inf -> 0
            const float p = exp2f(sc[hh] - mn);
            l[hh] = l[hh] * al + p;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[hh][e] = fmaf(p, vf[e], acc[hh][e] * al);
            m[hh] = mn;
          }
        }
      };
      const uint16_t* kg = op.kc + kvbase + sub * 8;
      const uint16_t* vg = op.vc + kvbase + sub * 8;
      for (int base = lo + cw * PPW; base < hi; base += NSTEP * CONSUMER_WARPS * PPW) {
        uint4 kv[NSTEP], vv[NSTEP];
#pragma unroll
        for (int u = 0; u < NSTEP; ++u) {
          const int t = base + u * CONSUMER_WARPS * PPW + grp;
          kv[u] = make_uint4(0, 0, 0, 0);
          vv[u] = make_uint4(0, 0, 0, 0);
          if (t < hi) {
            if (t == s) {
              kv[u] = *reinterpret_cast<const uint4*>(A.ks + sub * 8);
              vv[u] = *reinterpret_cast<const uint4*>(A.vs + sub * 8);
            } else {
              kv[u] = ldcg_u4(kg + (size_t)t * D);
              vv[u] = ldcg_u4(vg + (size_t)t * D);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < NSTEP; ++u) consume(kv[u], vv[u], base + u * CONSUMER_WARPS * PPW + grp < hi);
      }
      // merge the position groups of the warp
#pragma unroll
      for (int off = LP; off < 32; off <<= 1) {
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float mo = __shfl_xor_sync(0xffffffffu, m[hh], off);
          const float lo_ = __shfl_xor_sync(0xffffffffu, l[hh], off);
          const float mn = fmaxf(m[hh], mo);
          const float a = (mn == -INFINITY) ? 0.f : exp2f(m[hh] - mn);
          const float b = (mn == -INFINITY) ? 0.f : exp2f(mo - mn);
          l[hh] = l[hh] * a + lo_ * b;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float ao = __shfl_xor_sync(0xffffffffu, acc[hh][e], off);
            acc[hh][e] = acc[hh][e] * a + ao * b;
          }
          m[hh] = mn;
        }
      }
      if (grp == 0) {
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
#pragma unroll
          for (int e = 0; e < 8; ++e) A.wacc[cw][hh * D + sub * 8 + e] = acc[hh][e];
          if (sub == 0) {
            A.wm[cw][hh][0] = m[hh];
            A.wm[cw][hh][1] = l[hh];
          }
        }
      }
    }
    consumer_sync();
    // merge the warps in fixed order -> this chunk's partial.  Warps holding
    // (head, dim i): every warp on the CUDA-core path; on the tensor-core
    // path the NT warps whose 64 dims hold i (one per tile of a stage)
    constexpr int NT = STREAMED ? STAGE_BYTES / (4 * D) / 16 : CONSUMER_WARPS;
    for (int idx = ctid; idx < G * D; idx += CONSUMER_THREADS) {
      const int hh = idx / D, i = idx % D;
      const int w0 = STREAMED ? (i / 64) * NT : 0;
      float M = -INFINITY;
      for (int w = w0; w < w0 + NT; ++w) M = fmaxf(M, A.wm[w][hh][0]);
      float Ls = 0.f, Os = 0.f;
      if (M != -INFINITY) {
        for (int w = w0; w < w0 + NT; ++w) {
          const float f = exp2f(A.wm[w][hh][0] - M);
          Ls = fmaf(A.wm[w][hh][1], f, Ls);
          Os = fmaf(A.wacc[w][hh * D + i], f, Os);
        }
      }
      if (fused) {
        uint64_t* p = op.gpart + (((size_t)j * C + c) * G + hh) * (D + 2);
        st_tagged(p + 2 + i, Os, mytag);
        if (i == 0) {
          st_tagged(p, M, mytag);
          st_tagged(p + 1, Ls, mytag);
        }
      } else {
        float* p = const_cast<float*>(pbase) + ((size_t)hh * CS + c) * (D + 2);
        p[2 + i] = Os;
        if (i == 0) {
          p[0] = M;
          p[1] = Ls;
        }
      }
    }
  }
  if (fused) {
    if (c != 0 || !active) return true;
    // chunk 0 merges the group's chunks in chunk order once each partial
    // carries this iteration's tag (online rescaling, as for the split op):
    // all partial words are first gathered into shared memory, eight loads in
    // flight per thread, then merged from there
    float* pv = reinterpret_cast<float*>(&A);
    const int nwords = C * G * (D + 2);
    const uint64_t* pg = op.gpart + (size_t)j * nwords;
    bool mfail = false;
    consumer_sync();  // the chunk's own use of the scratch is over
    constexpr int GW = (MAX_GCHUNK * (MAX_G / 2) * (MAX_D + 2) + CONSUMER_THREADS - 1) / CONSUMER_THREADS;
    uint64_t w[GW];
    auto g_addr = [&](int u) { return pg + u * CONSUMER_THREADS + ctid; };
    auto g_valid = [&](int u) { return u * CONSUMER_THREADS + ctid < nwords; };
#pragma unroll
    for (int u = 0; u < GW; ++u) w[u] = g_valid(u) ? ld_tagged(g_addr(u)) : 0ull;
    mfail |= !settle_tagged(g, w, g_addr, g_valid, mytag, op.self, worker, (int)iter);
#pragma unroll
    for (int u = 0; u < GW; ++u)
      if (g_valid(u)) pv[u * CONSUMER_THREADS + ctid] = word_value(w[u]);
    if (consumer_sync_or(mfail)) return false;
    for (int idx = ctid; idx < G * D; idx += CONSUMER_THREADS) {
      const int hh = idx / D, i = idx % D;
      float M = -INFINITY, Ls = 0.f, Os = 0.f;
      for (int cc = 0; cc < C; ++cc) {
        const float* p = pv + ((size_t)cc * G + hh) * (D + 2);
        const float mc = p[0], lc = p[1], oc = p[2 + i];
        if (mc == -INFINITY) continue;
        if (mc > M) {
          const float sc = exp2f(M - mc);  // M = -inf -> 0
          Ls *= sc;
          Os *= sc;
          M = mc;
        }
        const float f = exp2f(mc - M);
        Ls = fmaf(lc, f, Ls);
        Os = fmaf(oc, f, Os);
      }
      st_tagged(op.a_out + (size_t)r * op.Hq * D + (size_t)(j * G + hh) * D + i, Os / Ls, mytag);
    }
    return !consumer_sync_or(mfail);
  }
  consumer_sync();
  if (ctid == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(op.merge_cnt + (size_t)r * Hkv + j, 1u);
    sm.last = (old + 1u) == (uint32_t)C;
    // the merging task restarts the count for the next iteration (whose
    // tasks depend on this merge's output)
    if (sm.last) atomicExch(op.merge_cnt + (size_t)r * Hkv + j, 0u);
  }
  consumer_sync();
  if (sm.last) {
    if (active) {
      __threadfence();
      // The chunk partials of the group's heads: first every chunk's (max,
      // sum) into shared memory and, per head, the weights exp2(m_c - M) and
      // the total sum; then each output element over the chunks in order,
      // eight loads in flight at a time (not one dependent round trip per
      // chunk).  The block merge's scratch is free again.
      float* mw = A.wacc[0];  // [G][C] maxima, then weights; [G][C] sums; [G] totals
      const int nml = G * C;
      for (int u = ctid; u < nml; u += CONSUMER_THREADS) {
        const float* p = pbase + ((size_t)(u / C) * CS + (u % C)) * (D + 2);
        mw[u] = __ldcg(p);
        mw[nml + u] = __ldcg(p + 1);
      }
      consumer_sync();
      if (ctid < G) {
        float M = -INFINITY, Ls = 0.f;
        for (int cc = 0; cc < C; ++cc) M = fmaxf(M, mw[ctid * C + cc]);
        for (int cc = 0; cc < C; ++cc) {
          const float mc = mw[ctid * C + cc];
          const float f = mc == -INFINITY ? 0.f : exp2f(mc - M);  // an empty chunk weighs 0
          mw[ctid * C + cc] = f;
          Ls = fmaf(mw[nml + ctid * C + cc], f, Ls);
        }
        mw[2 * nml + ctid] = Ls;
      }
      consumer_sync();
      for (int idx = ctid; idx < G * D; idx += CONSUMER_THREADS) {
        const int hh = idx / D, i = idx % D;
        const float* p = pbase + (size_t)hh * CS * (D + 2) + 2 + i;
        const float* wgt = mw + hh * C;
        float Os = 0.f;
        for (int c0 = 0; c0 < C; c0 += 8) {
          float ov[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) ov[u] = c0 + u < C ? __ldcg(p + (size_t)(c0 + u) * (D + 2)) : 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (c0 + u < C) Os = fmaf(ov[u], wgt[c0 + u], Os);
        }
        const float ov = Os / mw[2 * nml + hh];
        st_tagged(op.a_out + (size_t)r * op.Hq * D + (size_t)(j * G + hh) * D + i, ov, mytag);
        if (op.xb_out != nullptr) publish_xb_g(g, op, (j * G + hh) * D + i, r, ov);
      }
    } else {
      // an inactive request still publishes this iteration's version of its
      // output (zeros), which the next projection waits for
      for (int idx = ctid; idx < G * D; idx += CONSUMER_THREADS) {
        st_tagged(op.a_out + (size_t)r * op.Hq * D + (size_t)j * G * D + idx, 0.f, mytag);
        if (op.xb_out != nullptr) publish_xb_g(g, op, j * G * D + idx, r, 0.f);
      }
    }
    consumer_sync();
    if (ctid == 0) {
      if (op.xb_out != nullptr) {
        // the group's published rows, then their flag
        __threadfence();
        st_tagged(op.xf_out + (size_t)r * Hkv + j, 0.f, mytag);
      }
      red_release_add(g.events + (size_t)op.out_event * EVENT_STRIDE, 1u);
    }
  }
  return true;
}

// ------------------------------------------------------------------ embedding task
__device__ bool embed_task(const Graph& g, const OpDesc& op, int task, uint32_t iter, int ctid) {
  const int r = task;
  int s, q = 0;
  if (r < g.R && !request_state(g, r, iter, s, q)) {
    // inactive request (several requests, this one done): x carries this
    // iteration's version with zeros, so every reader's wait ends; nothing
    // of it reaches the request's tokens or cache
    const uint32_t mytag = vtag(g, iter, op.self);
    for (int i = ctid; i < op.N; i += CONSUMER_THREADS) st_tagged(op.x_out + (size_t)r * op.N + i, 0.f, mytag);
    if (op.xss_out != nullptr) {
      const int cw = ctid >> 5, lane = ctid & 31;
      for (int b = cw; b < op.xss_blocks; b += CONSUMER_WARPS) {
        if (op.xb_out != nullptr) {
          for (int i = b * BM + lane; i < min(op.N, (b + 1) * BM); i += 32) publish_xb_g(g, op, i, r, 0.f);
          __threadfence();
        }
        __syncwarp();
        if (lane == 0) st_tagged(op.xss_out + (size_t)b * g.R + r, 0.f, mytag);
      }
    }
    return true;
  }
  if (r < g.R) {
    const int64_t tok = __ldcg(g.tokens + (size_t)q * g.S + s);
    if (tok < 0 || tok >= g.V) {
      if (ctid == 0) record_error(g, -11 /*DEVICE*/, 8, -1, task, -1, (int)iter, (uint32_t)tok, (uint32_t)g.V);
      return true;
    }
    const uint16_t* row = op.table + (size_t)tok * op.N;
    uint64_t* x = op.x_out + (size_t)r * op.N;
    const uint32_t mytag = vtag(g, iter, op.self);
    const bool capture = (g.capture_iter == (int)iter) && g.cap_hidden != nullptr && op.capture_slot >= 0;
    for (int i = ctid * 8; i < op.N; i += CONSUMER_THREADS * 8) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + i));
      const float4 a = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
      const float4 b = make_float4(bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w));
      st_tagged(x + i + 0, a.x, mytag); st_tagged(x + i + 1, a.y, mytag);
      st_tagged(x + i + 2, a.z, mytag); st_tagged(x + i + 3, a.w, mytag);
      st_tagged(x + i + 4, b.x, mytag); st_tagged(x + i + 5, b.y, mytag);
      st_tagged(x + i + 6, b.z, mytag); st_tagged(x + i + 7, b.w, mytag);
      if (capture) {
        float* hc = g.cap_hidden + ((size_t)op.capture_slot * g.R + r) * g.H + i;
        *reinterpret_cast<float4*>(hc) = a;
        *reinterpret_cast<float4*>(hc + 4) = b;
      }
    }
    if (op.xss_out != nullptr) {
      // per-block sums of squares of the row (batched graphs): warp w takes
      // blocks w, w + 8, ..., lane l elements 4l..4l+3 of the block
      const int cw = ctid >> 5, lane = ctid & 31;
      for (int b = cw; b < op.xss_blocks; b += CONSUMER_WARPS) {
        float ss = 0.f;
        const int i = b * BM + lane * 4;
        if (i < op.N) {
          const uint2 w = __ldg(reinterpret_cast<const uint2*>(row + i));
          const float e0 = bf16_lo(w.x), e1 = bf16_hi(w.x), e2 = bf16_lo(w.y), e3 = bf16_hi(w.y);
          ss = e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
          if (op.xb_out != nullptr) {
            // the rows the next RMSNorm operation reads, before the sums
            publish_xb_g(g, op, i, r, e0); publish_xb_g(g, op, i + 1, r, e1);
            publish_xb_g(g, op, i + 2, r, e2); publish_xb_g(g, op, i + 3, r, e3);
          }
        }
        if (op.xb_out != nullptr) __threadfence();
        ss = warp_sum(ss);
        if (lane == 0) st_tagged(op.xss_out + (size_t)b * g.R + r, ss, mytag);
      }
    }
  }
  return true;
}

// ------------------------------------------------------------------ dispatch
// Attention dispatch by (G, D).  The fused projections + attention operation
// calls one non-inlined dispatch with every body inlined into it (the GEMV
// tasks' consumer loop then keeps its registers); the split-K operation calls
// a non-inlined function per (G, D), each with its own register allocation.
template <int G, int D, bool STREAMED>
__device__ __noinline__ bool attn_task_call(Smem& sm, const Graph& g, const OpDesc& op, int j, int c, int C, int r,
                                            int mode, int cw, int lane, uint32_t iter, int worker, uint32_t cstage) {
  return attn_task<G, D, STREAMED>(sm, g, op, j, c, C, r, mode, cw, lane, iter, worker, cstage);
}

__device__ __noinline__ bool attn_dispatch(Smem& sm, const Graph& g, const OpDesc& op, int j, int c, int C, int r,
                                           int mode, int cw, int lane, uint32_t iter, int worker) {
#define MPK_ATTN_CASE(GG, DD) \
  case GG * 1000 + DD: return attn_task<GG, DD, false>(sm, g, op, j, c, C, r, mode, cw, lane, iter, worker, 0u);
  switch (op.G * 1000 + op.d) {
    MPK_ATTN_CASE(1, 64) MPK_ATTN_CASE(2, 64) MPK_ATTN_CASE(4, 64)
    MPK_ATTN_CASE(1, 128) MPK_ATTN_CASE(2, 128) MPK_ATTN_CASE(4, 128)
    default: return false;
  }
#undef MPK_ATTN_CASE
}

__device__ __forceinline__ bool attn_dispatch_split(Smem& sm, const Graph& g, const OpDesc& op, int j, int c, int C,
                                                    int r, int mode, int cw, int lane, uint32_t iter, int worker,
                                                    uint32_t cstage) {
#define MPK_ATTN_CASE(GG, DD)                                                                                 \
  case GG * 1000 + DD:                                                                                        \
    return attn_task_call<GG, DD, true>(sm, g, op, j, c, C, r, mode, cw, lane, iter, worker, cstage);
  switch (op.G * 1000 + op.d) {
    MPK_ATTN_CASE(1, 64) MPK_ATTN_CASE(2, 64) MPK_ATTN_CASE(4, 64)
    MPK_ATTN_CASE(1, 128) MPK_ATTN_CASE(2, 128) MPK_ATTN_CASE(4, 128)
    default: return false;
  }
#undef MPK_ATTN_CASE
}

// A task of the split-K attention operation, its K/V streamed through the ring
// from stage cstage on.  Returns the stages it took, -1 on failure.  Not
// inlined, so the consumer loop keeps its registers.
__device__ __noinline__ int attn_split_task(Smem& sm, const Graph& g, const OpDesc& op, int task, uint32_t iter,
                                            int cw, int lane, int worker, uint32_t cstage) {
  int r, c, Cr;
  bool ok = true;
  if (attn_slot(g, op, task / op.Hkv, iter, r, c, Cr))
    ok = attn_dispatch_split(sm, g, op, task % op.Hkv, c, Cr, r, ATTN_SPLIT_OP, cw, lane, iter, worker, cstage);
  return ok ? (int)attn_stages(g, op, task, iter) : -1;
}

template <bool kStandalone, bool kBatch, bool kSplit, int BW>
__device__ void consumer_loop(Smem& sm, const Graph& g, int worker, int cw, int lane) {
  const int ctid = cw * 32 + lane;
  uint32_t fpos = 0, cstage = 0, accn = 0;
  while (true) {
    // fetch the next task entry (elected wait, shared decision)
    bool fail = false;
    if (ctid == 0) {
      const uint32_t f = fpos % TASK_FIFO;
      if (wait_mbar(g, &sm.fifo_full[f], (fpos / TASK_FIFO) & 1u, 4, worker)) {
        sm.cur_entry = sm.fifo[f];
        mbar_arrive(&sm.fifo_empty[f]);
      } else {
        fail = true;
      }
    }
    if (consumer_sync_or(fail)) return;
    const unsigned long long entry = sm.cur_entry;
    ++fpos;
    if (entry == QUEUE_TERMINATE) return;
    const uint32_t iter = (uint32_t)(entry >> 32);
    const int opi = (int)((entry >> 16) & 0xFFFFu);
    const int task = (int)(entry & 0xFFFFu);
    const OpDesc& op = g.ops[opi];

    uint64_t t_start = 0, t_ready = 0;
    if (g.profiling && ctid == 0) {
      t_start = globaltimer();
      sm.t_pro = 0ull;
      sm.t_data = 0ull;
      sm.t_stall = 0ull;
      sm.t_last = 0ull;
      sm.t_loop = 0ull;
    }
    // dependency: the event of the op this one follows
    if (!kStandalone && ctid == 0 && !op.tagged) {
      const uint32_t target = (iter + (uint32_t)op.dep_iter_offset) * (uint32_t)op.dep_trigger;
      if (target != 0 &&
          !wait_counter(g, g.events + (size_t)op.dep_event * EVENT_STRIDE, target, 1, opi, task, worker, (int)iter))
        fail = true;
    }
    if (g.profiling && ctid == 0) t_ready = globaltimer();
    if (consumer_sync_or(fail)) return;

    bool ok = true;
    if constexpr (kBatch) {
      switch (op.kind) {
        case TK_EMBED: ok = embed_task(g, op, task, iter, ctid); break;
        case TK_NORM_GEMV: ok = bgemm_task<TK_NORM_GEMV, BW>(sm, g, op, task, iter, cstage, accn, cw, lane, worker);
          bgemm_advance<BW>(op, task, cstage, accn); break;
        case TK_GEMV_RESID:
          ok = bgemm_task<TK_GEMV_RESID, BW>(sm, g, op, task, iter, cstage, accn, cw, lane, worker);
          bgemm_advance<BW>(op, task, cstage, accn);
          break;
        case TK_NORM_GEMV_SILU:
          ok = bgemm_task<TK_NORM_GEMV_SILU, BW>(sm, g, op, task, iter, cstage, accn, cw, lane, worker);
          bgemm_advance<BW>(op, task, cstage, accn);
          break;
        case TK_NORM_GEMV_ARGMAX:
          ok = bgemm_task<TK_NORM_GEMV_ARGMAX, BW>(sm, g, op, task, iter, cstage, accn, cw, lane, worker);
          bgemm_advance<BW>(op, task, cstage, accn);
          break;
        case TK_ATTN: {
          const int n = attn_split_task(sm, g, op, task, iter, cw, lane, worker, cstage);
          ok = n >= 0;
          cstage += ok ? (uint32_t)n : 0u;
          break;
        }
        default: ok = false;  // the fused projections + attention operation takes one request
      }
    } else switch (op.kind) {
      case TK_EMBED: ok = embed_task(g, op, task, iter, ctid); break;
      case TK_NORM_GEMV: ok = gemv_task<TK_NORM_GEMV>(sm, g, op, task, iter, cstage, cw, lane, worker); break;
      case TK_GEMV_RESID: ok = gemv_task<TK_GEMV_RESID>(sm, g, op, task, iter, cstage, cw, lane, worker); break;
      case TK_NORM_GEMV_SILU:
        ok = gemv_task<TK_NORM_GEMV_SILU>(sm, g, op, task, iter, cstage, cw, lane, worker);
        break;
      case TK_NORM_GEMV_ARGMAX:
        ok = gemv_task<TK_NORM_GEMV_ARGMAX>(sm, g, op, task, iter, cstage, cw, lane, worker);
        break;
      case TK_ATTN: {
        if constexpr (kSplit) {
          const int n = attn_split_task(sm, g, op, task, iter, cw, lane, worker, cstage);
          ok = n >= 0;
          cstage += ok ? (uint32_t)n : 0u;
        } else {
          ok = false;  // the host runs graphs with split-K attention on the kSplit kernels
        }
        break;
      }
      case TK_QKV_ATTN: ok = gemv_task<TK_QKV_ATTN>(sm, g, op, task, iter, cstage, cw, lane, worker); break;
      default: ok = false;
    }
    if (!ok) {
      if (ctid == 0) record_error(g, -11 /*DEVICE*/, 9, opi, task, worker, (int)iter, (uint32_t)op.kind, 0);
      return;  // uniform: every consumer thread takes the same branch
    }
    consumer_sync();
    if (ctid == 0) {
      // progress count for the scheduler's dispatch window (data readiness
      // travels with the tagged values, so no release is needed here)
      if (op.signal_per_task) red_relaxed_add(g.events + (size_t)op.out_event * EVENT_STRIDE, 1u);
      if (g.profiling) {
        const uint32_t k = atomicAdd(g.timeline_n, 1u);
        if (k < (uint32_t)g.max_timeline) {
          unsigned long long* rec = g.timeline + (size_t)k * TIMELINE_FIELDS;
          rec[0] = entry;
          rec[1] = (unsigned long long)worker;
          rec[2] = t_start;
          rec[3] = t_ready;
          rec[4] = globaltimer();
          rec[5] = sm.t_pro;
          rec[6] = sm.t_data;
          rec[7] = atomicAdd(&sm.fifo_t[(fpos - 1) % TASK_FIFO], 0ull);
          rec[8] = sm.t_stall;
          rec[9] = sm.t_last;
          rec[10] = sm.t_loop;
        }
      }
    }
  }
}

// ------------------------------------------------------------------ scheduler
__device__ void scheduler_lane(const Graph& g, int si, int lane) {
  const int wk = si + lane * g.num_sched;
  if (wk >= g.num_workers) return;
  if (!wait_counter(g, &g.ctl->ready, 1u, 7, -1, -1, wk, -1)) return;
  const uint32_t n_iter = __ldcg(&g.ctl->n_iter);
  uint32_t* qtail = g.q_tail + (size_t)wk * EVENT_STRIDE;
  const uint32_t* qhead = g.q_head + (size_t)wk * EVENT_STRIDE;
  unsigned long long* q = g.queue + (size_t)wk * QUEUE_CAP;
  uint32_t tail = 0, head_seen = 0;
  const int P = g.nops, W = g.num_workers;

  auto push = [&](unsigned long long e) -> bool {
    if (tail - head_seen >= (uint32_t)QUEUE_CAP) {
      if (!wait_counter(g, qhead, tail - QUEUE_CAP + 1, 6, -1, -1, wk, -1)) return false;
      head_seen = ld_acquire(qhead);
    }
    q[tail % QUEUE_CAP] = e;
    ++tail;
    st_release(qtail, tail);
    return true;
  };

  uint32_t off = 0;  // rotating task offset: op p's task t goes to worker (t + off) % W
  for (uint32_t n = 0; n < n_iter; ++n) {
    // host abort request, read once per iteration; the scheduler is ahead of
    // the workers by the dispatch window, so this read is off their path
    if (g.abort_flag != nullptr && *g.abort_flag != 0) {
      record_error(g, -10 /*ABORTED*/, 10, -1, -1, wk, (int)n, 0, 0);
      return;
    }
    if (aborted(g)) return;
    for (int p = 0; p < P; ++p) {
      const long long gidx = (long long)n * P + p - g.lookahead;
      if (g.lookahead > 0 && gidx >= 0) {
        const int pp = (int)(gidx % P);
        const uint32_t nn = (uint32_t)(gidx / P);
        const OpDesc& o = g.ops[pp];
        if (!wait_counter(g, g.events + (size_t)o.out_event * EVENT_STRIDE, (nn + 1u) * (uint32_t)o.out_trigger, 5,
                          pp, -1, wk, (int)nn))
          return;
      }
      if (g.ops[p].dynamic) {
        // every worker claims this op's tasks itself
        if (!push(pack_entry(n, (uint32_t)p, TASK_CLAIM))) return;
        continue;
      }
      const int nt = g.ops[p].ntasks;
      int t0 = ((wk - (int)off) % W + W) % W;
      for (int t = t0; t < nt; t += W)
        if (!push(pack_entry(n, (uint32_t)p, (uint32_t)t))) return;
      off = (off + (uint32_t)nt) % (uint32_t)W;
    }
  }
  push(QUEUE_TERMINATE);
}

// ------------------------------------------------------------------ kernels
// The ring's stages are released by every consumer warp (GEMV path) or by
// one MMA completion (tensor-core path).
template <bool kBatch>
__device__ __forceinline__ void init_barriers(Smem& sm) {
  sm.h_key = ~0ull;
  for (int i = 0; i < NSTAGES; ++i) {
    mbar_init(&sm.full[i], 1);
    mbar_init(&sm.empty[i], kBatch ? 1 : CONSUMER_WARPS);
  }
  for (int i = 0; i < NSLOT_MAX; ++i) {
    mbar_init(&sm.acc_full[i], 1);
    mbar_init(&sm.acc_empty[i], 4);
  }
  mbar_init(&sm.bfree, 1);
  sm.bfn = 0;
  mbar_init(&sm.bload, 1);
  sm.bload_n = 0;
  mbar_init(&sm.fin_bar, 1);
  for (int i = 0; i < TASK_FIFO; ++i) {
    mbar_init(&sm.fifo_full[i], 1);
    mbar_init(&sm.fifo_empty[i], 1);
  }
  fence_mbar_init();
}

// Dynamic shared memory: the layout plus slack to start it on a 1024-byte
// boundary (the swizzled tensor-core operands need that alignment).
extern __shared__ __align__(1024) uint8_t smem_raw[];
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;
static_assert(SMEM_BYTES <= 232448, "one worker block per SM: at most 227 KB of shared memory");

__device__ __forceinline__ Smem& smem_layout(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return *reinterpret_cast<Smem*>(raw + ((1024u - (a & 1023u)) & 1023u));
}

// A worker block: barriers (and, on the tensor-core path, the accumulator's
// tensor memory, allocated by consumer warp 0 and released by it after the
// last task, once no MMA is in flight), then the producer and consumer roles.
template <bool kStandalone, bool kBatch, bool kSplit, int BW = 8>
__device__ __forceinline__ void worker_block(Smem& sm, const Graph& g, int worker, uint32_t sa_iter, int sa_op) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) init_barriers<kBatch>(sm);
  if (kBatch && warp == PRODUCER_WARPS) tmem_alloc(&sm.tmem_base);
  if (kBatch) tc_fence_before_sync();
  __syncthreads();
  if (kBatch) tc_fence_after_sync();
  if (warp < PRODUCER_WARPS) {
    regs_dec<PRODUCER_REGS>();
    if (warp == 0 && lane == 0) producer_loop<kStandalone, kBatch, kSplit, BW>(sm, g, worker, sa_iter, sa_op);
    return;
  }
  regs_inc<CONSUMER_REGS>();
  consumer_loop<kStandalone, kBatch, kSplit, BW>(sm, g, worker, warp - PRODUCER_WARPS, lane);
  if (kBatch) {
    // the MMA-issuing thread waits (bounded) until none of its MMAs is outstanding
    if (warp == PRODUCER_WARPS + 4 && lane == 0) {
      mma_commit(&sm.fin_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sm.fin_bar, 0u) && globaltimer() - t0 < 200000000ull) {
      }
    }
    __syncwarp();
    tc_fence_before_sync();
    consumer_sync();
    tc_fence_after_sync();
    if (warp == PRODUCER_WARPS) tmem_dealloc(sm.tmem_base);
  }
}

template <bool kBatch, bool kSplit, int BW = 8>
__device__ __forceinline__ void persistent_body(const Graph& g) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if ((int)blockIdx.x < g.sched_ctas) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      // iterations of this run: the furthest any request still has to go;
      // prefill: every request's remaining positions, R per iteration, one
      // request after another
      uint32_t n_iter = 0;
      const int nq = g.prefill ? g.Rq : g.R;
      for (int q = 0; q < nq; ++q) {
        const int s = __ldcg(g.step + q);
        int end = g.S - 1;
        if (g.step_end != nullptr) end = min(end, __ldcg(g.step_end + q));
        const bool act = s >= 0 && s < end;
        const uint32_t left = act ? (uint32_t)(end - s) : 0u;
        if (g.prefill) {
          g.ctl->cum[q] = n_iter;
          n_iter += (left + (uint32_t)g.R - 1u) / (uint32_t)g.R;
        } else {
          n_iter = max(n_iter, left);
        }
        g.ctl->step0[q] = act ? s : -1;
        g.ctl->stop[q] = end;
      }
      if (g.prefill) g.ctl->cum[nq] = n_iter;
      g.ctl->n_iter = n_iter;
      st_release(&g.ctl->ready, 1u);
    }
    if (warp < SCHED_WARPS_PER_SM) {
      const int si = blockIdx.x * SCHED_WARPS_PER_SM + warp;
      if (si < g.num_sched) scheduler_lane(g, si, lane);
    }
    return;
  }
  worker_block<false, kBatch, kSplit, BW>(smem_layout(smem_raw), g, blockIdx.x - g.sched_ctas, 0, 0);
}

// Kernels: one request without split-K attention (the fused projections +
// attention operation), one request with it (long contexts), several requests
// (tensor-core projections, split-K attention): up to 8, and 9..16 (batch
// width 16).
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_persistent_kernel(const Graph g) {
  persistent_body<false, false>(g);
}
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_persistent_split_kernel(const Graph g) {
  persistent_body<false, true>(g);
}
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_persistent_batch_kernel(const Graph g) {
  persistent_body<true, true, 8>(g);
}
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_persistent_batch16_kernel(const Graph g) {
  persistent_body<true, true, 16>(g);
}

// One operation of one iteration as an ordinary launch: block b runs task b.
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_op_kernel(const Graph g, int op, uint32_t iter) {
  worker_block<true, false, false>(smem_layout(smem_raw), g, blockIdx.x, iter, op);
}
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_op_split_kernel(const Graph g, int op,
                                                                                  uint32_t iter) {
  worker_block<true, false, true>(smem_layout(smem_raw), g, blockIdx.x, iter, op);
}
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_op_batch_kernel(const Graph g, int op,
                                                                                  uint32_t iter) {
  worker_block<true, true, true, 8>(smem_layout(smem_raw), g, blockIdx.x, iter, op);
}
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_op_batch16_kernel(const Graph g, int op,
                                                                                    uint32_t iter) {
  worker_block<true, true, true, 16>(smem_layout(smem_raw), g, blockIdx.x, iter, op);
}

// ------------------------------------------------------------------ host-side launch helpers
size_t kernel_smem_bytes() { return SMEM_BYTES; }

cudaError_t prepare_kernels() {
  const void* ks[] = {(const void*)mpk_persistent_kernel,  (const void*)mpk_persistent_split_kernel,
                      (const void*)mpk_persistent_batch_kernel, (const void*)mpk_persistent_batch16_kernel,
                      (const void*)mpk_op_kernel, (const void*)mpk_op_split_kernel,
                      (const void*)mpk_op_batch_kernel, (const void*)mpk_op_batch16_kernel};
  for (const void* k : ks) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t max_blocks_per_sm(int* n) {
  const void* ks[] = {(const void*)mpk_persistent_kernel, (const void*)mpk_persistent_split_kernel,
                      (const void*)mpk_persistent_batch_kernel, (const void*)mpk_persistent_batch16_kernel};
  int m = 1 << 30;
  for (const void* k : ks) {
    int a = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&a, k, BLOCK_THREADS, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    m = a < m ? a : m;
  }
  *n = m;
  return cudaSuccess;
}

cudaError_t launch_persistent(const Graph& g, int grid, cudaStream_t stream) {
  void* args[] = {const_cast<Graph*>(&g)};
  const void* k = g.batched ? (g.bw > 8 ? (const void*)mpk_persistent_batch16_kernel
                                        : (const void*)mpk_persistent_batch_kernel)
                  : g.split_attn ? (const void*)mpk_persistent_split_kernel : (const void*)mpk_persistent_kernel;
  return cudaLaunchCooperativeKernel(k, dim3(grid), dim3(BLOCK_THREADS), args, SMEM_BYTES, stream);
}

// An operation whose tasks wait on one another (group mode) is launched
// cooperatively, so all of its blocks are resident together.
cudaError_t launch_op(const Graph& g, int op, int ntasks, uint32_t iter, bool cooperative, cudaStream_t stream) {
  const void* k = g.batched ? (g.bw > 8 ? (const void*)mpk_op_batch16_kernel : (const void*)mpk_op_batch_kernel)
                  : g.split_attn ? (const void*)mpk_op_split_kernel : (const void*)mpk_op_kernel;
  void* args[] = {const_cast<Graph*>(&g), &op, &iter};
  if (cooperative)
    return cudaLaunchCooperativeKernel(k, dim3(ntasks), dim3(BLOCK_THREADS), args, SMEM_BYTES, stream);
  return cudaLaunchKernel(k, dim3(ntasks), dim3(BLOCK_THREADS), args, SMEM_BYTES, stream);
}

}  // namespace mpk
