// Projections of a batch of requests on the tensor cores (tcgen05, sm_100a).
//
// With R = 2..MAX_BATCH requests in the graph, every projection of a decoding
// iteration is a dense contraction Y[R, N] = X[R, K] W^T ("Mirage Persistent
// Kernel: Fusing Multi-GPU LLM Inference into One Kernel Launch", section "How
// MPK Works": the same fused layers, now with several requests per step).
// Tasks form a grid of (row-block runs) x (reduction segments):
//
//  * producer: the weight tiles (BM rows x BK elements, 16 KB) come in by 2-D
//    tiled TMA copies with 128-byte swizzle, two tiles per ring stage, into
//    NSTB stages of the ring;
//  * consumers, prologue: the batch's input rows for the task's reduction
//    segment (after RMSNorm for the norm operations) are split into bf16
//    hi/lo pairs and written into the ring's remaining stages in the same
//    swizzled K-major layout: K block b at b * KBLOCK_BYTES, the hi rows as
//    BW / 8 eight-row atoms, the lo rows as as many more; request r's row at
//    128 r, its 16-byte chunk c at 16 (c ^ (r mod 8));
//  * one consumer thread issues the MMAs (M = BM weight rows, N = 2 BW columns,
//    K = 16 per instruction) into a tensor-memory accumulator and commits each
//    stage back to the producer;
//  * the first consumer warpgroup reads the accumulator (lane = weight row,
//    column = hi/lo input row), adds each request's hi and lo columns and runs
//    the operation's epilogue, or writes partial sums when the reduction is
//    split; the last segment task of a row block to arrive adds the partials
//    in segment order and runs the epilogue.
//
// Included by mpk_kernel.cu inside namespace mpk.

// Row blocks [rb0, rb1) and K blocks [kb0, kb1) of a task; seg is its
// reduction segment.  Task t computes segment t / ntb (of bsplit) for the run
// of row blocks [u nb / ntb, (u+1) nb / ntb), u = t mod ntb.
__device__ __forceinline__ void btask(const OpDesc& op, int task, int& rb0, int& rb1, int& kb0, int& kb1, int& seg) {
  seg = task / op.ntb;
  const int u = task - seg * op.ntb;
  rb0 = (int)(((long long)u * op.nb) / op.ntb);
  rb1 = (int)(((long long)(u + 1) * op.nb) / op.ntb);
  kb0 = (int)(((long long)seg * op.nkb) / op.bsplit);
  kb1 = (int)(((long long)(seg + 1) * op.nkb) / op.bsplit);
}

// A task's K blocks are processed in passes of at most MAX_KBLOCKS (the
// input rows held in shared memory): passes of the task's row blocks
// accumulate into one tensor-memory slot per block.
template <int BW>
__device__ __forceinline__ int bpasses(int nkbs) {
  return (nkbs + BGeo<BW>::MAX_KBLOCKS - 1) / BGeo<BW>::MAX_KBLOCKS;
}
__device__ __forceinline__ void bpass(int kb0, int kb1, int npass, int ps, int& kp0, int& kp1) {
  kp0 = kb0 + (int)(((long long)ps * (kb1 - kb0)) / npass);
  kp1 = kb0 + (int)(((long long)(ps + 1) * (kb1 - kb0)) / npass);
}

// Ring stages of one row block: gate/up take one K block of both matrices per
// stage, the other operations two K blocks of one matrix.
__device__ __forceinline__ int bstages(const OpDesc& op, int nkbs) {
  return op.kind == TK_NORM_GEMV_SILU ? nkbs : (nkbs + 1) / 2;
}

// Ring stages and accumulator slots a batched task takes.
template <int BW>
__device__ __forceinline__ void bgemm_counts(const OpDesc& op, int task, uint32_t& stages, uint32_t& blocks) {
  int rb0, rb1, kb0, kb1, seg;
  btask(op, task, rb0, rb1, kb0, kb1, seg);
  const int npass = bpasses<BW>(kb1 - kb0);
  uint32_t st = 0;
  for (int ps = 0; ps < npass; ++ps) {
    int kp0, kp1;
    bpass(kb0, kb1, npass, ps, kp0, kp1);
    st += (uint32_t)bstages(op, kp1 - kp0);
  }
  stages = st * (uint32_t)(rb1 - rb0);
  blocks = (uint32_t)(rb1 - rb0);
}

// Producer side of a batched task: its weight tiles, stage by stage.  False on
// abort or timeout.  t_issue (profiling) receives the first stage's issue time.
template <int BW>
__device__ bool bproduce(Smem& sm, const Graph& g, const OpDesc& op, int task, uint32_t& pstage, int worker,
                         uint64_t pol, unsigned long long* t_issue) {
  int rb0, rb1, kb0, kb1, seg;
  btask(op, task, rb0, rb1, kb0, kb1, seg);
  const bool pair = op.kind == TK_NORM_GEMV_SILU;
  const int npass = bpasses<BW>(kb1 - kb0);
  for (int ps = 0; ps < npass; ++ps) {
    int kp0, kp1;
    bpass(kb0, kb1, npass, ps, kp0, kp1);
    for (int rb = rb0; rb < rb1; ++rb) {
      const int row = rb * BM;
      const int s = pair ? 0 : seg_of(op, row);
      const int mrow = row - op.seg_row0[s];  // row within matrix s (rows past its end read as zeros)
      const void* tm = op.tmap[s];
      for (int kb = kp0; kb < kp1; kb += pair ? 1 : 2) {
        const uint32_t slot = pstage % NSTB;
        const uint32_t par = ((pstage / NSTB) & 1u) ^ 1u;
        if (!wait_mbar(g, &sm.empty[slot], par, 3, worker)) return false;
        if (t_issue != nullptr && ps == 0 && rb == rb0 && kb == kp0)
          atomicExch(t_issue, (unsigned long long)globaltimer());
        const int nbox = pair ? 2 : min(2, kp1 - kb);
        mbar_arrive_expect_tx(&sm.full[slot], (uint32_t)(nbox * BOX_BYTES));
        tma_load_2d(sm.ring[slot], tm, kb * BK, mrow, &sm.full[slot], pol);
        if (pair) tma_load_2d(sm.ring[slot] + BOX_BYTES, op.tmap_up, kb * BK, mrow, &sm.full[slot], pol);
        else if (nbox == 2) tma_load_2d(sm.ring[slot] + BOX_BYTES, tm, (kb + 1) * BK, mrow, &sm.full[slot], pol);
        ++pstage;
      }
    }
  }
  return true;
}

// Epilogue of output row `row` for every request: v[r] is the row's dot
// product with request r's input (gate/up: v gate, u up).  RESID leaves the
// new residual values in nx (0 for rows past the end), for the block's sums
// of squares.
template <int KIND, int BW>
__device__ __forceinline__ void bepilogue(const Graph& g, const OpDesc& op, int row, const float* v, const float* u,
                                          uint32_t iter, uint32_t xtag, uint32_t mytag, bool capture,
                                          unsigned long long (&best)[BW], float (&nx)[BW],
                                          bool& fail, int worker) {
  const int R = g.R;
  if (KIND == TK_NORM_GEMV) {
    const int s = seg_of(op, row);
    const int local = row - op.seg_row0[s], ns = op.grp_rows[s];
#pragma unroll
    for (int r = 0; r < BW; ++r)
      if (r < R) st_tagged(op.y[s] + (size_t)r * ns + local, v[r], mytag);
  } else if (KIND == TK_GEMV_RESID) {
    uint64_t w[BW];
#pragma unroll
    for (int r = 0; r < BW; ++r) w[r] = r < R ? ld_tagged(op.x_out + (size_t)r * op.N + row) : 0ull;
#pragma unroll
    for (int r = 0; r < BW; ++r) {
      if (r < R) {
        uint64_t* p = op.x_out + (size_t)r * op.N + row;
        if (word_tag(w[r]) != xtag) {
          w[r] = poll_word(g, p, xtag, op.self, worker, (int)iter);
          fail |= word_tag(w[r]) != xtag;
        }
        nx[r] = word_value(w[r]) + v[r];
        st_tagged(p, nx[r], mytag);
        if (capture && op.capture_slot >= 0 && g.cap_hidden != nullptr)
          g.cap_hidden[((size_t)op.capture_slot * R + r) * g.H + row] = nx[r];
      }
    }
  } else if (KIND == TK_NORM_GEMV_SILU) {
#pragma unroll
    for (int r = 0; r < BW; ++r) {
      if (r < R) {
        nx[r] = silu_f(v[r]) * u[r];
        st_tagged(op.a_out + (size_t)r * op.N + row, nx[r], mytag);
      }
    }
  } else {  // LM head
#pragma unroll
    for (int r = 0; r < BW; ++r) {
      if (r < R) {
        const unsigned long long key = argmax_key(v[r], (uint32_t)row);
        best[r] = key > best[r] ? key : best[r];
        if (capture && g.cap_logits != nullptr) g.cap_logits[(size_t)r * g.V + row] = v[r];
      }
    }
  }
}

// Element k of request r's input row into the next projection's published
// input rows of batch width BW: bf16 hi/lo of x (times w_next[k] when the
// next operation is an RMSNorm) at row r (hi) and BW + r (lo) of K block
// k / 64, 16-byte chunk (k mod 64) / 8 swizzled by r mod 8.
template <int BW>
__device__ __forceinline__ void publish_xb(const OpDesc& op, int k, int r, float x) {
  const float h = op.xb_w != nullptr ? x * __uint_as_float((uint32_t)op.xb_w[k] << 16) : x;
  const uint16_t hi = f32_to_bf16_rn(h);
  const uint16_t lo = f32_to_bf16_rn(h - __uint_as_float((uint32_t)hi << 16));
  uint16_t* blk = op.xb_out + (size_t)(k >> 6) * (BGeo<BW>::KBLOCK_BYTES / 2);
  const int off = r * BK + ((((k & 63) >> 3) ^ (r & 7)) << 3) + (k & 7);
  blk[off] = hi;
  blk[BW * BK + off] = lo;
}
// The same for a writer outside the contractions (embedding, attention
// merge), at the graph's batch width.
__device__ __forceinline__ void publish_xb_g(const Graph& g, const OpDesc& op, int k, int r, float x) {
  if (g.bw > 8) publish_xb<16>(op, k, r, x);
  else publish_xb<8>(op, k, r, x);
}

// Two bf16 (bits) in one word, element k in the low half.
__device__ __forceinline__ uint32_t pack2(uint16_t a, uint16_t b) { return (uint32_t)a | ((uint32_t)b << 16); }

// hi = bf16(v) and lo = bf16(v - hi) of eight values (v - hi is exact in fp32).
__device__ __forceinline__ void split8(const float (&v)[8], uint4& hi, uint4& lo) {
  uint16_t h[8], l[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    h[e] = f32_to_bf16_rn(v[e]);
    l[e] = f32_to_bf16_rn(v[e] - __uint_as_float((uint32_t)h[e] << 16));
  }
  hi = make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]), pack2(h[4], h[5]), pack2(h[6], h[7]));
  lo = make_uint4(pack2(l[0], l[1]), pack2(l[2], l[3]), pack2(l[4], l[5]), pack2(l[6], l[7]));
}

// Consumer side of a batched task (all CONSUMER_THREADS threads).  cstage and
// accn are the ring stage and accumulator use the task starts at (the caller
// advances them by bgemm_counts).  Roles inside the task: consumer warp MMA_WARP's lane 0
// issues every row block's MMAs, alternating between two tensor-memory
// accumulators; warps 0..3 (tensor-memory lanes 0..127, one weight row per
// thread) read each accumulator as soon as it is complete and run the
// epilogue, so the next block's MMAs overlap it.
//
// Not inlined: the task gets its own register allocation, so neither its
// arrays nor the attention's are spilled around the other.
template <int KIND, int BW>
__device__ __noinline__ bool bgemm_task(Smem& sm, const Graph& g, const OpDesc& op, int task, uint32_t iter,
                                        uint32_t cstage, uint32_t accn, int cw, int lane, int worker) {
  constexpr bool PAIR = KIND == TK_NORM_GEMV_SILU;
  constexpr bool NORM = KIND != TK_GEMV_RESID;
  constexpr int MMA_WARP = 4;
  constexpr int BN = BGeo<BW>::BN, KBB = BGeo<BW>::KBLOCK_BYTES, NSLOT = BGeo<BW>::NSLOT;
  const int ctid = cw * 32 + lane;
  const int R = g.R;
  int rb0, rb1, kb0, kb1, seg;
  btask(op, task, rb0, rb1, kb0, kb1, seg);
  const int nblk = rb1 - rb0;
  const int npass = bpasses<BW>(kb1 - kb0);
  const bool split = op.bsplit > 1;
  uint8_t* bsm = sm.ring[NSTB];
  const uint32_t xtag = vtag(g, iter, op.x_writer) + op.tag_skew;
  const uint32_t atag = vtag(g, iter, op.a_writer) + op.tag_skew;
  const uint32_t mytag = vtag(g, iter, op.self);
  const uint64_t* src = NORM ? op.x : op.a_in;
  const uint32_t stag = NORM ? xtag : atag;
  const uint32_t tmem = sm.tmem_base;
  const int nrows = op.N;
  // partial sums: [segment][row][PW] floats, PW = the requests' values (gate/up:
  // then the up values), so a thread moves its row with 16-byte accesses
  constexpr int PW = PAIR ? 2 * BW : BW;
  const size_t SEGW = (size_t)nrows * PW;
  bool fail = false;
  unsigned long long best[BW];
#pragma unroll
  for (int r = 0; r < BW; ++r) best[r] = 0ull;

  // ---- RMSNorm factor of every request from the per-block sums of squares
  // its writer published (warp w: requests w, w + 8, ..., blocks in a fixed order)
  if (NORM) {
    bool pfail = false;
    for (int rq = cw; rq < R; rq += CONSUMER_WARPS) {
      float ss = 0.f;
      for (int b = lane; b < op.xss_blocks; b += 32) {
        const uint64_t* p = op.xss_in + (size_t)b * R + rq;
        uint64_t w = ld_tagged(p);
        if (word_tag(w) != stag) {
          w = poll_word(g, p, stag, op.self, worker, (int)iter);
          pfail |= word_tag(w) != stag;
        }
        ss += word_value(w);
      }
      ss = warp_sum(ss);
      if (lane == 0) sm.brinv[rq] = 1.0f / sqrtf(ss / (float)op.K + op.eps);
      if (op.xb_in != nullptr) __threadfence();  // acquire: the rows published before these sums
    }
    if (consumer_sync_or(pfail)) return false;
  }

  // ---- published plain inputs: the tagged flags covering this task's K range
  // (each thread acquires what it observed; the barrier hands it on)
  if (!NORM && op.xb_in != nullptr) {
    bool pfail = false;
    const int g0 = kb0 * BK / op.xf_grp, g1 = min(kb1 * BK - 1, op.K - 1) / op.xf_grp;
    const int ng = g1 - g0 + 1, nq = ng * (op.xf_rstride != 0 ? R : 1);
    for (int q = ctid; q < nq; q += CONSUMER_THREADS) {
      const uint64_t* p = op.xf_in + (size_t)(q / ng) * op.xf_rstride + g0 + q % ng;
      uint64_t w = ld_tagged(p);
      if (word_tag(w) != stag) {
        w = poll_word(g, p, stag, op.self, worker, (int)iter);
        pfail |= word_tag(w) != stag;
      }
      __threadfence();
    }
    if (consumer_sync_or(pfail)) return false;
  }

  for (int ps = 0; ps < npass; ++ps) {
    int kp0, kp1;
    bpass(kb0, kb1, npass, ps, kp0, kp1);
    const int nkbs = kp1 - kp0;
    const int nst = bstages(op, nkbs);
    const bool last = ps == npass - 1;
    if (ps > 0) {
      // the previous pass's MMAs are done reading the input rows
      bool ok = true;
      if (ctid == 0) {
        ok = wait_mbar(g, &sm.bfree, sm.bfn & 1u, 3, worker);
        ++sm.bfn;
      }
      if (consumer_sync_or(fail || !ok)) return false;
    }
    const bool published = op.xb_in != nullptr;
    if (published) {
      // the writers' published rows (released before the sums of squares or
      // flags acquired above): one bulk copy of this pass's K blocks, waited
      // for by the MMA-issuing thread
      if (ctid == 0) {
        fence_acq_rel_gpu();
        fence_proxy_async_global();
        const uint32_t bytes = (uint32_t)nkbs * (uint32_t)KBB;
        mbar_arrive_expect_tx(&sm.bload, bytes);
        bulk_g2s(bsm, op.xb_in + (size_t)kp0 * (KBB / 2), bytes, &sm.bload, policy_evict_first());
      }
      consumer_sync();
    } else {
    // ---- the input rows of this pass's K blocks as bf16 hi/lo pairs into
    // the swizzled layout; FL chunks of 8 elements per thread in flight
    {
      bool pfail = false;
      const int nch = nkbs * 8;  // 16-byte chunks per request row
      const int total = BW * nch;
      constexpr int FL = 2;
      for (int q0 = ctid; q0 < total; q0 += FL * CONSUMER_THREADS) {
        uint64_t w[FL][8];
#pragma unroll
        for (int u = 0; u < FL; ++u) {
          const int q = q0 + u * CONSUMER_THREADS;
          const int r = q / nch;
          if (q < total && r < R) {
            const uint64_t* p = src + (size_t)r * op.K + (size_t)kp0 * BK + (size_t)(q - r * nch) * 8;
#pragma unroll
            for (int e = 0; e < 8; e += 2) ld_tagged2(p + e, w[u][e], w[u][e + 1]);
          }
        }
#pragma unroll
        for (int u = 0; u < FL; ++u) {
          const int q = q0 + u * CONSUMER_THREADS;
          if (q < total) {
            const int r = q / nch, cc = q - r * nch;
            const int kbl = cc >> 3, ch = cc & 7;
            uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi;
            if (r < R) {
              const int k = kp0 * BK + cc * 8;
              const uint64_t* p = src + (size_t)r * op.K + k;
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                if (word_tag(w[u][e]) != stag) {
                  w[u][e] = poll_word(g, p + e, stag, op.self, worker, (int)iter);
                  pfail |= word_tag(w[u][e]) != stag;
                }
                v[e] = word_value(w[u][e]);
              }
              if (NORM) {
                const uint4 nw = __ldg(reinterpret_cast<const uint4*>(op.norm_w + k));
                const float ri = sm.brinv[r];
                v[0] = v[0] * ri * bf16_lo(nw.x); v[1] = v[1] * ri * bf16_hi(nw.x);
                v[2] = v[2] * ri * bf16_lo(nw.y); v[3] = v[3] * ri * bf16_hi(nw.y);
                v[4] = v[4] * ri * bf16_lo(nw.z); v[5] = v[5] * ri * bf16_hi(nw.z);
                v[6] = v[6] * ri * bf16_lo(nw.w); v[7] = v[7] * ri * bf16_hi(nw.w);
              }
              split8(v, hi, lo);
            }
            uint8_t* dst = bsm + kbl * KBB + r * (BK * 2) + ((ch ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(dst) = hi;
            *reinterpret_cast<uint4*>(dst + KBB / 2) = lo;
          }
        }
      }
      fence_proxy_async_smem();  // the tensor cores read these bytes next
      if (consumer_sync_or(pfail)) return false;
    }
    }
    if (ps == 0 && g.profiling && ctid == 0) sm.t_pro = globaltimer();

    if (cw == MMA_WARP) {
      // ---- MMAs of this pass for every row block: block i accumulates in
      // slot (accn + i) mod NSLOT, handed to the epilogue after the last pass
      if (lane == 0) {
        const uint32_t idesc = mma_idesc_bf16(BM, BN);
        bool ok = true;
        if (published) {
          ok = wait_mbar(g, &sm.bload, sm.bload_n & 1u, 3, worker);
          if (!ok) {  // never leave the block with the copy in flight
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&sm.bload, sm.bload_n & 1u) && globaltimer() - t0 < 200000000ull) {
            }
          }
          ++sm.bload_n;
        }
        for (int i = 0; i < nblk; ++i) {
          const uint32_t a = accn + (uint32_t)i, slot = a % NSLOT, use = a / NSLOT;
          // the epilogue has read this slot's previous block
          if (ps == 0 && ok) ok = wait_mbar(g, &sm.acc_empty[slot], (use & 1u) ^ 1u, 3, worker);
          tc_fence_after_sync();
          const uint32_t dacc = tmem + slot * (uint32_t)(2 * BN);
          for (int st = 0; ok && st < nst; ++st) {
            const uint32_t cs = cstage + (uint32_t)(i * nst + st);
            const uint32_t rs = cs % NSTB;
            const uint64_t w0 = g.profiling ? globaltimer() : 0ull;
            ok = wait_mbar(g, &sm.full[rs], (cs / NSTB) & 1u, 3, worker);
            if (g.profiling) {
              const uint64_t w1 = globaltimer();
              sm.t_stall += w1 - w0;
              sm.t_last = w1;
              if (ps == 0 && i == 0 && st == 0) sm.t_data = w1;
            }
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t a0 = smem_u32(sm.ring[rs]);
            if (PAIR) {
              const uint32_t b0 = smem_u32(bsm) + (uint32_t)st * KBB;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                const uint64_t bd = sw128_desc(b0 + kk * 32);
                const uint32_t acc = (ps | st | kk) != 0;
                mma_bf16_ss(dacc, sw128_desc(a0 + kk * 32), bd, idesc, acc);
                mma_bf16_ss(dacc + BN, sw128_desc(a0 + BOX_BYTES + kk * 32), bd, idesc, acc);
              }
            } else {
              const int nbox = min(2, nkbs - 2 * st);
              for (int b = 0; b < nbox; ++b) {
                const uint32_t b0 = smem_u32(bsm) + (uint32_t)(2 * st + b) * KBB;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                  mma_bf16_ss(dacc, sw128_desc(a0 + b * BOX_BYTES + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                              (ps | st | b | kk) != 0);
              }
            }
            mma_commit(&sm.empty[rs]);  // the stage returns to the producer once these MMAs have read it
          }
          if (last) mma_commit(&sm.acc_full[slot]);  // also after a failure: it ends the epilogue's wait
        }
        if (!last) mma_commit(&sm.bfree);  // also after a failure: it ends the next pass's wait
        fail |= !ok;
      }
      __syncwarp();
    } else if (cw < 4 && last) {
      // ---- epilogue of every row block, in order, as soon as its slot is complete
      const bool capture = (g.capture_iter == (int)iter);
      const uint32_t lanes = (uint32_t)(cw * 32) << 16;
      for (int i = 0; i < nblk; ++i) {
        const int rb = rb0 + i;
        const uint32_t a = accn + (uint32_t)i, slot = a % NSLOT, use = a / NSLOT;
        bool ok = true;
        if (lane == 0) ok = wait_mbar(g, &sm.acc_full[slot], use & 1u, 3, worker);
        ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
        tc_fence_after_sync();
        float d[BN], du[BN];
        const uint32_t dacc = tmem + slot * (uint32_t)(2 * BN) + lanes;
        tmem_ld_cols<BN>(dacc, d);
        if (PAIR) tmem_ld_cols<BN>(dacc + BN, du);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.acc_empty[slot]);
        fail |= !ok;
        // W hi + W lo per request (published rows: times the request's RMS factor)
        float v[BW], u[BW], nx[BW];
#pragma unroll
        for (int r = 0; r < BW; ++r) {
          v[r] = d[r] + d[BW + r];
          u[r] = PAIR ? du[r] + du[BW + r] : 0.f;
          if (NORM && published) {
            v[r] *= sm.brinv[r];
            u[r] *= sm.brinv[r];
          }
          nx[r] = 0.f;
        }
        const int row = rb * BM + cw * 32 + lane;
        bool finish = !split;  // this task runs the block's epilogue
        if (split) {
          if (ok && row < nrows) {
            float4* pp = reinterpret_cast<float4*>(op.bpart + (size_t)seg * SEGW + (size_t)row * PW);
#pragma unroll
            for (int c4 = 0; c4 < BW / 4; ++c4) {
              pp[c4] = make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
              if (PAIR) pp[BW / 4 + c4] = make_float4(u[4 * c4], u[4 * c4 + 1], u[4 * c4 + 2], u[4 * c4 + 3]);
            }
          }
          // The last segment task of this row block to arrive adds the
          // partial sums in segment order and runs the epilogue.  (Thread 0's
          // acquire-release arrival, then the barrier, order the other tasks'
          // partials before every thread's reads.)
          epi_sync();
          if (ctid == 0) {
            const uint32_t old = atom_add_acq_rel(op.blk_cnt + rb, 1u);
            sm.blast = ((old + 1u) % (uint32_t)op.bsplit) == 0u;
          }
          epi_sync();
          finish = sm.blast != 0;
          if (finish && row < nrows) {
            constexpr int V4 = PW / 4;  // float4 per partial row
            const float4* base = reinterpret_cast<const float4*>(op.bpart + (size_t)row * PW);
            const size_t seg4 = SEGW / 4;
            // segments in pairs, both segments' loads issued first
            for (int s0 = 0; s0 < op.bsplit; s0 += 2) {
              float4 q[2][V4];
#pragma unroll
              for (int j = 0; j < 2; ++j)
                if (s0 + j < op.bsplit)
#pragma unroll
                  for (int c4 = 0; c4 < V4; ++c4) q[j][c4] = __ldcg(base + (size_t)(s0 + j) * seg4 + c4);
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                if (s0 + j < op.bsplit) {
                  const float* f = reinterpret_cast<const float*>(q[j]);
#pragma unroll
                  for (int r = 0; r < BW; ++r) {
                    v[r] = (s0 + j) == 0 ? f[r] : v[r] + f[r];
                    if (PAIR) u[r] = (s0 + j) == 0 ? f[BW + r] : u[r] + f[BW + r];
                  }
                }
              }
            }
          }
        }
        if (finish) {
          if (ok && row < nrows)
            bepilogue<KIND, BW>(g, op, row, v, u, iter, xtag, mytag, capture, best, nx, fail, worker);
          if ((KIND == TK_GEMV_RESID || KIND == TK_NORM_GEMV_SILU) && op.xb_out != nullptr && row < nrows) {
#pragma unroll
            for (int r = 0; r < BW; ++r)
              if (r < R) publish_xb<BW>(op, row, r, nx[r]);
          }
          if (KIND == TK_NORM_GEMV_SILU && op.xb_out != nullptr) {
            // the row block's flag, after all its rows
            epi_sync();
            if (ctid == 0) {
              __threadfence();
              st_tagged(op.xf_out + rb, 0.f, mytag);
            }
          }
          if (KIND == TK_GEMV_RESID && op.xss_out != nullptr) {
            // the block's sums of squares of the new x, per request: lanes,
            // then warps 0..3 in order
#pragma unroll
            for (int r = 0; r < BW; ++r) {
              const float ssr = warp_sum(nx[r] * nx[r]);
              if (lane == 0) sm.bss[i & 1][cw][r] = ssr;
            }
            epi_sync();
            if (ctid < R) {
              const float t = sm.bss[i & 1][0][ctid] + sm.bss[i & 1][1][ctid] + sm.bss[i & 1][2][ctid] +
                              sm.bss[i & 1][3][ctid];
              if (op.xb_out != nullptr) __threadfence();  // the block's published rows first
              st_tagged(op.xss_out + (size_t)rb * R + ctid, t, mytag);
            }
          }
        }
      }
    }
    cstage += (uint32_t)(nblk * nst);
  }
  if (consumer_sync_or(fail)) return false;
  if (g.profiling && ctid == 0) sm.t_loop = globaltimer();

  if (KIND == TK_NORM_GEMV_ARGMAX) {
    // per-request maxima of the task -> one 64-bit atomicMax each; the last
    // task of the operation to arrive writes the tokens
    if (cw < 4) {
#pragma unroll
      for (int r = 0; r < BW; ++r) {
        const unsigned long long b = warp_max_u64(best[r]);
        if (lane == 0) sm.bbest[cw][r] = b;
      }
    }
    consumer_sync();
    if (ctid == 0) {
      for (int r = 0; r < R; ++r) {
        unsigned long long b = 0ull;
        for (int w = 0; w < 4; ++w) b = sm.bbest[w][r] > b ? sm.bbest[w][r] : b;
        if (b != 0ull) atomicMax(op.keys + r, b);
      }
      __threadfence();
      const uint32_t old = atomicAdd(op.arrive, 1u);
      sm.last = ((old + 1u) % (uint32_t)op.ntasks) == 0u;
    }
    consumer_sync();
    argmax_tokens(sm, g, op, iter, ctid);
  }
  return true;
}
