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
};
static_assert(MAX_G * MAX_D / 2 >= 512, "attention scratch");

struct GemvScratch {
  float red[2][MAX_RPS][MAX_KW][2];              // per-row partial dots [parity][row][k-warp][gate/up]
};

struct __align__(128) Smem {
  uint8_t ring[NSTAGES][STAGE_BYTES];
  union {
    AttnScratch a;
    GemvScratch g;
  } u;
  float ss[CONSUMER_WARPS];
  unsigned long long bestk[CONSUMER_WARPS];
  unsigned long long fifo[TASK_FIFO];
  uint64_t full[NSTAGES];
  uint64_t empty[NSTAGES];
  uint64_t fifo_full[TASK_FIFO];
  uint64_t fifo_empty[TASK_FIFO];
  unsigned long long cur_entry;
  int32_t last;     // last-arrival flag
};

// ------------------------------------------------------------------ status / waits
__device__ __forceinline__ bool aborted(const Graph& g) {
  if (ld_volatile_i32(&g.status->code) != 0) return true;
  return false;
}

__device__ __noinline__ void record_error(const Graph& g, int code, int where, int op, int task,
                                          int worker, int iter, uint32_t observed, uint32_t expected) {
  if (atomicCAS(&g.status->code, 0, code) == 0) {
    g.status->where = where;
    g.status->op = op;
    g.status->task = task;
    g.status->worker = worker;
    g.status->iter = iter;
    g.status->observed = observed;
    g.status->expected = expected;
    __threadfence();
  }
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

// ------------------------------------------------------------------ task geometry
__device__ __forceinline__ void task_rows(const OpDesc& op, int task, int& row0, int& row1) {
  row0 = (int)(((long long)task * op.N) / op.ntasks);
  row1 = (int)(((long long)(task + 1) * op.N) / op.ntasks);
}

__device__ __forceinline__ bool is_gemv(int kind) {
  return kind == TK_NORM_GEMV || kind == TK_GEMV_RESID || kind == TK_NORM_GEMV_SILU ||
         kind == TK_NORM_GEMV_ARGMAX;
}

__device__ __forceinline__ bool request_active(const Graph& g, int r, int& s) {
  s = __ldcg(g.step + r);
  int end = g.S - 1;
  if (g.step_end != nullptr) {
    int e = __ldcg(g.step_end + r);
    end = e < end ? e : end;
  }
  return s >= 0 && s < end;
}

// Locate global row `row` of a stacked multi-matrix operation.
__device__ __forceinline__ int seg_of(const OpDesc& op, int row) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < MAX_SEG; ++i)
    if (i < op.nseg && row >= op.seg_row0[i]) s = i;
  return s;
}

// ------------------------------------------------------------------ producer
// Issue the bulk copies of one stage: rows [r, r+n) of the op's row space.
__device__ void issue_stage(const OpDesc& op, int r, int n, uint8_t* dst, uint64_t* bar, uint64_t pol) {
  const uint32_t row_bytes = (uint32_t)op.K * 2u;
  if (op.kind == TK_NORM_GEMV_SILU) {
    bulk_g2s(dst, op.W[0] + (size_t)r * op.K, row_bytes * n, bar, pol);
    bulk_g2s(dst + (size_t)op.rps * row_bytes, op.W_up + (size_t)r * op.K, row_bytes * n, bar, pol);
    return;
  }
  while (n > 0) {
    const int s = seg_of(op, r);
    const int seg_end = op.seg_row0[s + 1];
    const int cnt = min(n, seg_end - r);
    bulk_g2s(dst, op.W[s] + (size_t)(r - op.seg_row0[s]) * op.K, row_bytes * cnt, bar, pol);
    dst += (size_t)cnt * row_bytes;
    r += cnt;
    n -= cnt;
  }
}

template <bool kStandalone>
__device__ void producer_loop(Smem& sm, const Graph& g, int worker, uint32_t sa_iter, int sa_op) {
  const uint64_t pol = policy_evict_first();
  uint32_t qpos = 0, fpos = 0, pstage = 0;
  bool ok = true;
  uint32_t* qtail = g.q_tail + (size_t)worker * EVENT_STRIDE;
  uint32_t* qhead = g.q_head + (size_t)worker * EVENT_STRIDE;
  while (true) {
    unsigned long long entry;
    if (kStandalone) {
      entry = (fpos == 0) ? pack_entry(sa_iter, (uint32_t)sa_op, blockIdx.x) : QUEUE_TERMINATE;
    } else {
      if (!wait_counter(g, qtail, qpos + 1, 2, -1, -1, worker, -1)) { ok = false; break; }
      entry = __ldcg(g.queue + (size_t)worker * QUEUE_CAP + (qpos % QUEUE_CAP));
      ++qpos;
      st_release(qhead, qpos);
    }
    const uint32_t f = fpos % TASK_FIFO;
    if (!wait_mbar(g, &sm.fifo_empty[f], ((fpos / TASK_FIFO) & 1u) ^ 1u, 4, worker)) { ok = false; break; }
    sm.fifo[f] = entry;
    mbar_arrive(&sm.fifo_full[f]);
    ++fpos;
    if (entry == QUEUE_TERMINATE) break;

    const int opi = (int)((entry >> 16) & 0xFFFFu);
    const int task = (int)(entry & 0xFFFFu);
    const OpDesc& op = g.ops[opi];
    if (!is_gemv(op.kind)) continue;
    int row0, row1;
    task_rows(op, task, row0, row1);
    const uint32_t bytes_row = (uint32_t)op.K * 2u * (op.kind == TK_NORM_GEMV_SILU ? 2u : 1u);
    for (int r = row0; r < row1; r += op.rps) {
      const int n = min(op.rps, row1 - r);
      const uint32_t slot = pstage % NSTAGES;
      if (!wait_mbar(g, &sm.empty[slot], ((pstage / NSTAGES) & 1u) ^ 1u, 3, worker)) { ok = false; break; }
      mbar_arrive_expect_tx(&sm.full[slot], bytes_row * (uint32_t)n);
      issue_stage(op, r, n, sm.ring[slot], &sm.full[slot], pol);
      ++pstage;
    }
    if (!ok) break;
  }
  if (!ok) {
    // Never leave the block with bulk copies in flight: wait (bounded) for the
    // most recent stages to land before returning.
    const uint32_t first = pstage > (uint32_t)NSTAGES ? pstage - NSTAGES : 0u;
    for (uint32_t s = first; s < pstage; ++s) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sm.full[s % NSTAGES], (s / NSTAGES) & 1u)) {
        if (globaltimer() - t0 > 200000000ull) break;
      }
    }
  }
}

// ------------------------------------------------------------------ consumer helpers
// Elected-thread wait for a ring stage.  Returns true on failure (thread 0
// only); the caller shares the outcome through consumer_sync_or.
__device__ __forceinline__ bool stage_wait_elected(Smem& sm, const Graph& g, uint32_t cstage, int ctid,
                                                   int worker) {
  if (ctid != 0) return false;
  const uint32_t slot = cstage % NSTAGES;
  return !wait_mbar(g, &sm.full[slot], (cstage / NSTAGES) & 1u, 3, worker);
}

template <int EPL>
__device__ __forceinline__ float dot_slice(const uint16_t* w, const float (&h)[EPL], int lane) {
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int j = 0; j < EPL / 8; ++j) {
    const uint4 v = *reinterpret_cast<const uint4*>(w + j * 256 + lane * 8);
    a0 = fmaf(bf16_lo(v.x), h[j * 8 + 0], a0);
    a1 = fmaf(bf16_hi(v.x), h[j * 8 + 1], a1);
    a0 = fmaf(bf16_lo(v.y), h[j * 8 + 2], a0);
    a1 = fmaf(bf16_hi(v.y), h[j * 8 + 3], a1);
    a0 = fmaf(bf16_lo(v.z), h[j * 8 + 4], a0);
    a1 = fmaf(bf16_hi(v.z), h[j * 8 + 5], a1);
    a0 = fmaf(bf16_lo(v.w), h[j * 8 + 6], a0);
    a1 = fmaf(bf16_hi(v.w), h[j * 8 + 7], a1);
  }
  return a0 + a1;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

// ------------------------------------------------------------------ GEMV tasks
// Rows [row0,row1) of W (bf16, [rows, K] row-major) against one input vector.
// Consumer warp cw covers K slice kwi = cw % kw for rows i = grp (mod rw),
// grp = cw / kw; each lane holds EPL elements of h in registers.  Per stage
// every warp writes its per-row partial dot into shared memory; after the
// stage barrier the first n threads sum the kw partials in fixed order and run
// the operation's epilogue.
template <int KIND, int EPL>
__device__ bool gemv_task(Smem& sm, const Graph& g, const OpDesc& op, int task, uint32_t iter,
                          uint32_t& cstage, int cw, int lane, int worker) {
  const int ctid = cw * 32 + lane;
  const int K = op.K, kw = op.kw, rw = op.rw, rps = op.rps;
  const bool computes = cw < op.nwarps;
  const int kwi = cw % kw, grp = cw / kw;
  const int kbase = kwi * (K / kw);
  int row0, row1;
  task_rows(op, task, row0, row1);

  // ---- prologue: the input vector slice of this warp, rounded to bf16
  float h[EPL];
  if (KIND == TK_GEMV_RESID) {
#pragma unroll
    for (int j = 0; j < EPL / 8; ++j) {
      const uint4 a = ldcg_u4(op.a_in + kbase + j * 256 + lane * 8);
      h[j * 8 + 0] = bf16_lo(a.x); h[j * 8 + 1] = bf16_hi(a.x);
      h[j * 8 + 2] = bf16_lo(a.y); h[j * 8 + 3] = bf16_hi(a.y);
      h[j * 8 + 4] = bf16_lo(a.z); h[j * 8 + 5] = bf16_hi(a.z);
      h[j * 8 + 6] = bf16_lo(a.w); h[j * 8 + 7] = bf16_hi(a.w);
    }
  } else {
    // RMSNorm statistics over the whole input (fixed reduction order).
    float ss = 0.f;
    for (int k = ctid * 4; k < K; k += CONSUMER_THREADS * 4) {
      const float4 v = ldcg_f4(op.x + k);
      ss = fmaf(v.x, v.x, ss); ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss); ss = fmaf(v.w, v.w, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) sm.ss[cw] = ss;
    consumer_sync();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < CONSUMER_WARPS; ++w) tot += sm.ss[w];
    const float rinv = 1.0f / sqrtf(tot / (float)K + op.eps);
#pragma unroll
    for (int j = 0; j < EPL / 8; ++j) {
      const int k = kbase + j * 256 + lane * 8;
      const float4 x0 = ldcg_f4(op.x + k), x1 = ldcg_f4(op.x + k + 4);
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(op.norm_w + k));
      h[j * 8 + 0] = round_bf16(x0.x * rinv * bf16_lo(w.x));
      h[j * 8 + 1] = round_bf16(x0.y * rinv * bf16_hi(w.x));
      h[j * 8 + 2] = round_bf16(x0.z * rinv * bf16_lo(w.y));
      h[j * 8 + 3] = round_bf16(x0.w * rinv * bf16_hi(w.y));
      h[j * 8 + 4] = round_bf16(x1.x * rinv * bf16_lo(w.z));
      h[j * 8 + 5] = round_bf16(x1.y * rinv * bf16_hi(w.z));
      h[j * 8 + 6] = round_bf16(x1.z * rinv * bf16_lo(w.w));
      h[j * 8 + 7] = round_bf16(x1.w * rinv * bf16_hi(w.w));
    }
  }

  unsigned long long best = 0ull;
  const bool capture = (g.capture_iter == (int)iter);
  int par = 0;
  // first stage
  if (row0 < row1 && consumer_sync_or(stage_wait_elected(sm, g, cstage, ctid, worker))) return false;
  for (int r = row0; r < row1; r += rps) {
    const int n = min(rps, row1 - r);
    const uint32_t slot = cstage % NSTAGES;
    const uint8_t* stage = sm.ring[slot];
    if (computes) {
      for (int i0 = grp; i0 < n; i0 += 4 * rw) {
        float acc[4], accu[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = i0 + q * rw;
          acc[q] = 0.f;
          accu[q] = 0.f;
          if (i < n) {
            const uint16_t* wrow = reinterpret_cast<const uint16_t*>(stage + (size_t)i * K * 2) + kbase;
            acc[q] = dot_slice<EPL>(wrow, h, lane);
            if (KIND == TK_NORM_GEMV_SILU) {
              const uint16_t* urow =
                  reinterpret_cast<const uint16_t*>(stage + (size_t)(rps + i) * K * 2) + kbase;
              accu[q] = dot_slice<EPL>(urow, h, lane);
            }
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[q] = warp_sum(acc[q]);
          if (KIND == TK_NORM_GEMV_SILU) accu[q] = warp_sum(accu[q]);
        }
        if (lane == 0) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = i0 + q * rw;
            if (i < n) {
              sm.u.g.red[par][i][kwi][0] = acc[q];
              if (KIND == TK_NORM_GEMV_SILU) sm.u.g.red[par][i][kwi][1] = accu[q];
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[slot]);
    ++cstage;
    // Wait for the next stage of this task while the others reach the barrier.
    const bool fail = (r + rps < row1) && stage_wait_elected(sm, g, cstage, ctid, worker);
    const bool stop = consumer_sync_or(fail);
    // ---- epilogue of this stage
    if (ctid < n) {
      float v = 0.f, u = 0.f;
      for (int kk = 0; kk < kw; ++kk) {
        v += sm.u.g.red[par][ctid][kk][0];
        if (KIND == TK_NORM_GEMV_SILU) u += sm.u.g.red[par][ctid][kk][1];
      }
      const int row = r + ctid;
      if (KIND == TK_NORM_GEMV) {
        const int s = seg_of(op, row);
        op.y[s][row - op.seg_row0[s]] = v;
      } else if (KIND == TK_GEMV_RESID) {
        const float nx = __ldcg(op.x_out + row) + v;
        op.x_out[row] = nx;
        if (capture && op.capture_slot >= 0 && g.cap_hidden != nullptr)
          g.cap_hidden[(size_t)op.capture_slot * g.R * g.H + row] = nx;
      } else if (KIND == TK_NORM_GEMV_SILU) {
        op.a_out[row] = f32_to_bf16_rn(silu_f(v) * u);
      } else {  // LM head
        const unsigned long long key = argmax_key(v, (uint32_t)row);
        best = key > best ? key : best;
        if (capture && g.cap_logits != nullptr) g.cap_logits[row] = v;
      }
    }
    par ^= 1;
    if (stop) return false;
  }

  if (KIND == TK_NORM_GEMV_ARGMAX) {
    // Per-task maximum -> one 64-bit atomicMax; the last task to arrive
    // finishes the iteration.
    best = warp_max_u64(best);
    if (lane == 0) sm.bestk[cw] = best;
    consumer_sync();
    if (ctid == 0) {
      unsigned long long b = 0ull;
      for (int w = 0; w < CONSUMER_WARPS; ++w) b = sm.bestk[w] > b ? sm.bestk[w] : b;
      atomicMax(op.keys, b);
      __threadfence();
      const uint32_t old = atomicAdd(op.arrive, 1u);
      sm.last = ((old + 1u) % (uint32_t)op.ntasks) == 0u;
    }
    consumer_sync();
    if (sm.last) {
      __threadfence();
      if (ctid < g.R) {
        const int rq = ctid;
        int s;
        if (request_active(g, rq, s)) {
          const unsigned long long key = atomicAdd(op.keys + rq, 0ull);
          const int64_t nxt = (int64_t)argmax_key_index(key);
          int64_t* trow = g.tokens + (size_t)rq * g.S;
          if (__ldcg(trow + s + 1) == -1) trow[s + 1] = nxt;
          if (op.pred != nullptr) op.pred[(size_t)rq * g.S + s + 1] = nxt;
          g.step[rq] = s + 1;
        }
        op.keys[rq] = 0ull;
      }
      consumer_sync();
      if (ctid == 0) {
        __threadfence();
        red_release_add(g.events + (size_t)op.out_event * EVENT_STRIDE, 1u);
      }
    }
  }
  return true;
}

// ------------------------------------------------------------------ attention task
// Task (kv head j, chunk c, request r).  Prologue: RMSNorm over the head dim and
// rotate-half RoPE of the G query heads of the group and of k; the last chunk
// appends bf16 k, v at position s.  Main loop: LP = D/8 lanes per position (8
// dims per lane), 32/LP positions per warp step, online softmax in base 2 per
// query head.  Partials (max, sum, unnormalised output) go to global memory;
// the last chunk task of (r, j) to arrive merges them in chunk order and
// writes o = bf16(output).
template <int G, int D>
__device__ bool attn_task(Smem& sm, const Graph& g, const OpDesc& op, int task, int cw, int lane) {
  constexpr int LP = D / 8;          // lanes per position
  constexpr int PPW = 32 / LP;       // positions per warp step
  constexpr float LOG2E = 1.4426950408889634f;
  const int ctid = cw * 32 + lane;
  const int Hkv = op.Hkv, C = op.C;
  const int j = task % Hkv;
  const int c = (task / Hkv) % C;
  const int r = task / (Hkv * C);
  int s;
  const bool active = request_active(g, r, s);
  AttnScratch& A = sm.u.a;
  const size_t kvbase = ((((size_t)op.layer * g.R + r) * Hkv + j) * (size_t)op.S) * D;
  const float* pbase = op.part + (((size_t)r * op.Hq + (size_t)j * G) * C) * (D + 2);

  if (active) {
    const int npos = s + 1;
    const int lo = (int)(((long long)c * npos) / C);
    const int hi = (int)(((long long)(c + 1) * npos) / C);
    // ---- prologue: rows 0..G-1 = query heads, G = k, G+1 = v
    for (int row = cw; row < G + 2; row += CONSUMER_WARPS) {
      constexpr int EL = D / 32;  // elements per lane
      float x[EL];
      const float* src = row < G ? op.q + (size_t)r * op.Hq * D + (size_t)(j * G + row) * D
                       : row == G ? op.k + (size_t)r * Hkv * D + (size_t)j * D
                                  : op.v + (size_t)r * Hkv * D + (size_t)j * D;
#pragma unroll
      for (int e = 0; e < EL; ++e) x[e] = __ldcg(src + lane + 32 * e);
      if (row <= G) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < EL; ++e) ss = fmaf(x[e], x[e], ss);
        ss = warp_sum(ss);
        const float rinv = 1.0f / sqrtf(ss / (float)D + op.eps);
        const uint16_t* wn = row < G ? op.qn_w : op.kn_w;
#pragma unroll
        for (int e = 0; e < EL; ++e) {
          const uint16_t wb = __ldg(wn + lane + 32 * e);
          x[e] = x[e] * rinv * __uint_as_float((uint32_t)wb << 16);
        }
        // rotate-half RoPE: element i pairs with i + D/2 (same lane, e + EL/2)
        const float2* cs = op.rope + (size_t)s * (D / 2);
#pragma unroll
        for (int e = 0; e < EL / 2; ++e) {
          const float2 t = __ldg(cs + lane + 32 * e);
          const float a = x[e], b = x[e + EL / 2];
          x[e] = a * t.x - b * t.y;
          x[e + EL / 2] = b * t.x + a * t.y;
        }
      }
#pragma unroll
      for (int e = 0; e < EL; ++e) {
        const int i = lane + 32 * e;
        if (row < G) A.qs[row * D + i] = x[e];
        else if (row == G) A.ks[i] = f32_to_bf16_rn(x[e]);
        else A.vs[i] = f32_to_bf16_rn(x[e]);
      }
    }
    consumer_sync();
    if (c == C - 1 && ctid < D / 4) {
      // append k (first D/8 threads) and v (next D/8) at position s: 16 B each
      const int half = D / 8;
      const int which = ctid / half, q8 = ctid % half;
      uint16_t* dst = (which == 0 ? op.kc : op.vc) + kvbase + (size_t)s * D + q8 * 8;
      const uint16_t* srcs = (which == 0 ? A.ks : A.vs) + q8 * 8;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(srcs);
    }

    // ---- main loop
    const int grp = lane / LP, sub = lane % LP;
    const float qscale = LOG2E / sqrtf((float)D);
    float qr[G][8], acc[G][8], m[G], l[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      m[hh] = -INFINITY;
      l[hh] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        qr[hh][e] = A.qs[hh * D + sub * 8 + e] * qscale;
        acc[hh][e] = 0.f;
      }
    }
    const uint16_t* kg = op.kc + kvbase + sub * 8;
    const uint16_t* vg = op.vc + kvbase + sub * 8;
    for (int base = lo + cw * PPW; base < hi; base += CONSUMER_WARPS * PPW) {
      const int t = base + grp;
      const bool valid = t < hi;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (valid) {
        if (t == s) {
          kv = *reinterpret_cast<const uint4*>(A.ks + sub * 8);
          vv = *reinterpret_cast<const uint4*>(A.vs + sub * 8);
        } else {
          kv = ldcg_u4(kg + (size_t)t * D);
          vv = ldcg_u4(vg + (size_t)t * D);
        }
      }
      const float kf[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
                           bf16_lo(kv.z), bf16_hi(kv.z), bf16_lo(kv.w), bf16_hi(kv.w)};
      float sc[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(qr[hh][e], kf[e], a);
#pragma unroll
        for (int o = 1; o < LP; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        sc[hh] = a;
      }
      if (valid) {
        const float vf[8] = {bf16_lo(vv.x), bf16_hi(vv.x), bf16_lo(vv.y), bf16_hi(vv.y),
                             bf16_lo(vv.z), bf16_hi(vv.z), bf16_lo(vv.w), bf16_hi(vv.w)};
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
    consumer_sync();
    // merge the warps in fixed order -> this chunk's partial
    for (int idx = ctid; idx < G * D; idx += CONSUMER_THREADS) {
      const int hh = idx / D, i = idx % D;
      float M = -INFINITY;
      for (int w = 0; w < CONSUMER_WARPS; ++w) M = fmaxf(M, A.wm[w][hh][0]);
      float Ls = 0.f, Os = 0.f;
      if (M != -INFINITY) {
        for (int w = 0; w < CONSUMER_WARPS; ++w) {
          const float f = exp2f(A.wm[w][hh][0] - M);
          Ls = fmaf(A.wm[w][hh][1], f, Ls);
          Os = fmaf(A.wacc[w][hh * D + i], f, Os);
        }
      }
      float* p = const_cast<float*>(pbase) + ((size_t)hh * C + c) * (D + 2);
      p[2 + i] = Os;
      if (i == 0) {
        p[0] = M;
        p[1] = Ls;
      }
    }
  }
  consumer_sync();
  if (ctid == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(op.merge_cnt + (size_t)r * Hkv + j, 1u);
    sm.last = ((old + 1u) % (uint32_t)C) == 0u;
  }
  consumer_sync();
  if (sm.last) {
    if (active) {
      __threadfence();
      for (int idx = ctid; idx < G * D; idx += CONSUMER_THREADS) {
        const int hh = idx / D, i = idx % D;
        const float* p = pbase + (size_t)hh * C * (D + 2);
        float M = -INFINITY;
        for (int cc = 0; cc < C; ++cc) M = fmaxf(M, __ldcg(p + (size_t)cc * (D + 2)));
        float Ls = 0.f, Os = 0.f;
        for (int cc = 0; cc < C; ++cc) {
          const float mc = __ldcg(p + (size_t)cc * (D + 2));
          const float f = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
          Ls = fmaf(__ldcg(p + (size_t)cc * (D + 2) + 1), f, Ls);
          Os = fmaf(__ldcg(p + (size_t)cc * (D + 2) + 2 + i), f, Os);
        }
        op.a_out[(size_t)r * op.Hq * D + (size_t)(j * G + hh) * D + i] = f32_to_bf16_rn(Os / Ls);
      }
    }
    consumer_sync();
    if (ctid == 0) {
      __threadfence();
      red_release_add(g.events + (size_t)op.out_event * EVENT_STRIDE, 1u);
    }
  }
  return true;
}

// ------------------------------------------------------------------ embedding task
__device__ bool embed_task(const Graph& g, const OpDesc& op, int task, uint32_t iter, int ctid) {
  const int r = task;
  int s;
  if (r < g.R && request_active(g, r, s)) {
    const int64_t tok = __ldcg(g.tokens + (size_t)r * g.S + s);
    if (tok < 0 || tok >= g.V) {
      if (ctid == 0) record_error(g, -11 /*DEVICE*/, 8, -1, task, -1, (int)iter, (uint32_t)tok, (uint32_t)g.V);
      return true;
    }
    const uint16_t* row = op.table + (size_t)tok * op.N;
    float* x = op.x_out + (size_t)r * op.N;
    const bool capture = (g.capture_iter == (int)iter) && g.cap_hidden != nullptr && op.capture_slot >= 0;
    for (int i = ctid * 8; i < op.N; i += CONSUMER_THREADS * 8) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + i));
      const float4 a = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
      const float4 b = make_float4(bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w));
      *reinterpret_cast<float4*>(x + i) = a;
      *reinterpret_cast<float4*>(x + i + 4) = b;
      if (capture) {
        float* hc = g.cap_hidden + ((size_t)op.capture_slot * g.R + r) * g.H + i;
        *reinterpret_cast<float4*>(hc) = a;
        *reinterpret_cast<float4*>(hc + 4) = b;
      }
    }
  }
  return true;
}

// ------------------------------------------------------------------ dispatch
template <int KIND>
__device__ bool gemv_dispatch(Smem& sm, const Graph& g, const OpDesc& op, int task, uint32_t iter,
                              uint32_t& cstage, int cw, int lane, int worker) {
  switch (op.epl) {
    case 8: return gemv_task<KIND, 8>(sm, g, op, task, iter, cstage, cw, lane, worker);
    case 16: return gemv_task<KIND, 16>(sm, g, op, task, iter, cstage, cw, lane, worker);
    case 24: return gemv_task<KIND, 24>(sm, g, op, task, iter, cstage, cw, lane, worker);
    case 32: return gemv_task<KIND, 32>(sm, g, op, task, iter, cstage, cw, lane, worker);
    case 48: return gemv_task<KIND, 48>(sm, g, op, task, iter, cstage, cw, lane, worker);
    case 64: return gemv_task<KIND, 64>(sm, g, op, task, iter, cstage, cw, lane, worker);
    default: return false;
  }
}

__device__ bool attn_dispatch(Smem& sm, const Graph& g, const OpDesc& op, int task, int cw, int lane) {
  const int key = op.G * 1000 + op.d;
  switch (key) {
    case 1000 + 64: return attn_task<1, 64>(sm, g, op, task, cw, lane);
    case 2000 + 64: return attn_task<2, 64>(sm, g, op, task, cw, lane);
    case 4000 + 64: return attn_task<4, 64>(sm, g, op, task, cw, lane);
    case 1000 + 128: return attn_task<1, 128>(sm, g, op, task, cw, lane);
    case 2000 + 128: return attn_task<2, 128>(sm, g, op, task, cw, lane);
    case 4000 + 128: return attn_task<4, 128>(sm, g, op, task, cw, lane);
    default: return false;
  }
}

template <bool kStandalone>
__device__ void consumer_loop(Smem& sm, const Graph& g, int worker, int cw, int lane) {
  const int ctid = cw * 32 + lane;
  uint32_t fpos = 0, cstage = 0;
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
    if (g.profiling && ctid == 0) t_start = globaltimer();
    // dependency: the event of the op this one follows
    if (!kStandalone && ctid == 0) {
      const uint32_t target = (iter + (uint32_t)op.dep_iter_offset) * (uint32_t)op.dep_trigger;
      if (target != 0 &&
          !wait_counter(g, g.events + (size_t)op.dep_event * EVENT_STRIDE, target, 1, opi, task, worker, (int)iter))
        fail = true;
    }
    if (g.profiling && ctid == 0) t_ready = globaltimer();
    if (consumer_sync_or(fail)) return;

    bool ok = true;
    switch (op.kind) {
      case TK_EMBED: ok = embed_task(g, op, task, iter, ctid); break;
      case TK_NORM_GEMV: ok = gemv_dispatch<TK_NORM_GEMV>(sm, g, op, task, iter, cstage, cw, lane, worker); break;
      case TK_GEMV_RESID: ok = gemv_dispatch<TK_GEMV_RESID>(sm, g, op, task, iter, cstage, cw, lane, worker); break;
      case TK_NORM_GEMV_SILU:
        ok = gemv_dispatch<TK_NORM_GEMV_SILU>(sm, g, op, task, iter, cstage, cw, lane, worker);
        break;
      case TK_NORM_GEMV_ARGMAX:
        ok = gemv_dispatch<TK_NORM_GEMV_ARGMAX>(sm, g, op, task, iter, cstage, cw, lane, worker);
        break;
      case TK_ATTN: ok = attn_dispatch(sm, g, op, task, cw, lane); break;
      default: ok = false;
    }
    if (!ok) {
      if (ctid == 0) record_error(g, -11 /*DEVICE*/, 9, opi, task, worker, (int)iter, (uint32_t)op.kind, 0);
      return;  // uniform: every consumer thread takes the same branch
    }
    consumer_sync();
    if (ctid == 0) {
      if (op.signal_per_task) {
        __threadfence();
        red_release_add(g.events + (size_t)op.out_event * EVENT_STRIDE, 1u);
      }
      if (g.profiling) {
        const uint32_t k = atomicAdd(g.timeline_n, 1u);
        if (k < (uint32_t)g.max_timeline) {
          unsigned long long* rec = g.timeline + (size_t)k * 5;
          rec[0] = entry;
          rec[1] = (unsigned long long)worker;
          rec[2] = t_start;
          rec[3] = t_ready;
          rec[4] = globaltimer();
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
__device__ __forceinline__ void init_barriers(Smem& sm) {
  for (int i = 0; i < NSTAGES; ++i) {
    mbar_init(&sm.full[i], 1);
    mbar_init(&sm.empty[i], CONSUMER_WARPS);
  }
  for (int i = 0; i < TASK_FIFO; ++i) {
    mbar_init(&sm.fifo_full[i], 1);
    mbar_init(&sm.fifo_empty[i], 1);
  }
  fence_mbar_init();
}

extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_persistent_kernel(const Graph g) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if ((int)blockIdx.x < g.sched_ctas) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      // iterations of this run: the furthest any request still has to go
      uint32_t n_iter = 0;
      for (int r = 0; r < g.R; ++r) {
        int s;
        if (request_active(g, r, s)) {
          int end = g.S - 1;
          if (g.step_end != nullptr) end = min(end, __ldcg(g.step_end + r));
          n_iter = max(n_iter, (uint32_t)(end - s));
        }
      }
      g.ctl->n_iter = n_iter;
      st_release(&g.ctl->ready, 1u);
    }
    if (warp < SCHED_WARPS_PER_SM) {
      const int si = blockIdx.x * SCHED_WARPS_PER_SM + warp;
      if (si < g.num_sched) scheduler_lane(g, si, lane);
    }
    return;
  }

  const int worker = blockIdx.x - g.sched_ctas;
  if (threadIdx.x == 0) init_barriers(sm);
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) producer_loop<false>(sm, g, worker, 0, 0);
    return;
  }
  consumer_loop<false>(sm, g, worker, warp - 1, lane);
}

// One operation of one iteration as an ordinary launch: block b runs task b.
extern "C" __global__ void __launch_bounds__(BLOCK_THREADS, 1) mpk_op_kernel(const Graph g, int op, uint32_t iter) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) init_barriers(sm);
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) producer_loop<true>(sm, g, blockIdx.x, iter, op);
    return;
  }
  consumer_loop<true>(sm, g, blockIdx.x, warp - 1, lane);
}

// ------------------------------------------------------------------ host-side launch helpers
size_t kernel_smem_bytes() { return sizeof(Smem); }

cudaError_t prepare_kernels() {
  cudaError_t e = cudaFuncSetAttribute(mpk_persistent_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(Smem));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(mpk_op_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem));
}

cudaError_t max_blocks_per_sm(int* n) {
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, mpk_persistent_kernel, BLOCK_THREADS, sizeof(Smem));
}

cudaError_t launch_persistent(const Graph& g, int grid, cudaStream_t stream) {
  void* args[] = {const_cast<Graph*>(&g)};
  return cudaLaunchCooperativeKernel((const void*)mpk_persistent_kernel, dim3(grid), dim3(BLOCK_THREADS), args,
                                     sizeof(Smem), stream);
}

cudaError_t launch_op(const Graph& g, int op, int ntasks, uint32_t iter, cudaStream_t stream) {
  mpk_op_kernel<<<ntasks, BLOCK_THREADS, sizeof(Smem), stream>>>(g, op, iter);
  return cudaGetLastError();
}

}  // namespace mpk
