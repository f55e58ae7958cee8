// Internal layout shared by the host compiler and the device runtime.
#pragma once
#include <stdint.h>

#include "mpk.h"

namespace mpk {

// Worker block: a producer warpgroup (its warp 0 streams the weights, the
// other three only hand their registers over) + CONSUMER_WARPS compute warps
// in two warpgroups.  The launch gives every thread LAUNCH_REGS registers;
// setmaxnreg then moves them from the producer warpgroup to the consumers.
constexpr int CONSUMER_WARPS = 8;
constexpr int CONSUMER_THREADS = CONSUMER_WARPS * 32;
constexpr int PRODUCER_WARPS = 4;
constexpr int BLOCK_THREADS = CONSUMER_THREADS + PRODUCER_WARPS * 32;
constexpr int LAUNCH_REGS = 168;    // 65536 / 384 threads, rounded down to a multiple of 8
constexpr int PRODUCER_REGS = 56;
constexpr int CONSUMER_REGS = 224;
static_assert(PRODUCER_WARPS * 32 * PRODUCER_REGS + CONSUMER_THREADS * CONSUMER_REGS <= BLOCK_THREADS * LAUNCH_REGS,
              "register hand-over must stay within the launch's registers");
#ifndef MPK_STAGE_BYTES
#define MPK_STAGE_BYTES 32768
#endif
#ifndef MPK_NSTAGES
#define MPK_NSTAGES 6
#endif
constexpr int STAGE_BYTES = MPK_STAGE_BYTES;  // one weight stage in shared memory
constexpr int NSTAGES = MPK_NSTAGES;          // weight ring depth
constexpr int TASK_FIFO = 4;                // decoded task entries buffered per worker
constexpr int QUEUE_CAP = 64;               // global task queue entries per worker
constexpr int MAX_RPS = 64;                 // rows per stage upper bound
constexpr int MAX_K = 4096;                 // longest GEMV input kept in shared memory (fp32);
                                            // longer residual projections are split (ksplit)
static_assert(MAX_K % 256 == 0, "the permuted input layout works in blocks of 256");
static_assert(MAX_K == MPK_MAX_GEMV_K, "the header states the input buffer length");
constexpr int MAX_NORM_K = 4096;            // longest RMSNorm input (held in registers)
constexpr int MAX_XS = 1024;                // residual rows of a task preloaded to shared memory
constexpr int MAX_SEG = 3;
constexpr int MAX_KSPLIT = 8;               // reduction segments of one split residual projection
constexpr int MAX_G = 8;                    // query heads per kv head
constexpr int MAX_D = 128;                  // head dim
constexpr int MAX_GCHUNK = 8;               // fused op: attention chunks per kv head (tasks 0.. of the group)
constexpr int MAX_SPLIT_CHUNKS = 256;       // split-K op: chunks per (request, kv head) (the merge's weights fit the scratch)
constexpr int SCHED_WARPS_PER_SM = 4;

// Tensor-core path (an operation over 2..MAX_BATCH requests): every
// projection is a dense contraction [R, K] x W^T computed by tcgen05 MMAs of
// M = BM weight rows x N columns, K in blocks of BK elements.  The fp32 input
// of request r is split into two bf16 rows, hi = bf16(h) in column r and
// lo = bf16(h - hi) in column BW + r, so one MMA yields W hi + W lo: the
// contraction sees the input to about 16 significant bits, with the weights
// exact.  BW, the batch width, is 8 for up to 8 requests and 16 for 9..16
// (N = 2 BW = 16 or 32, both valid shapes for M = 128).  Weights arrive as
// BM x BK tiles (TMA, 128-byte swizzle); the input rows are held in the ring's
// last stages in the same layout (BW / 8 eight-row swizzle atoms of hi rows,
// then as many of lo rows, per K block); accumulators live in tensor memory.
constexpr int MAX_BATCH = 16;               // requests of one contraction
constexpr int MAX_PREFILL = 8;              // positions of a prefill graph's iteration
constexpr int BM = 128;                     // weight rows per MMA (tensor-memory lanes)
constexpr int BK = 64;                      // K elements per tile row (128 bytes)
constexpr int BOX_BYTES = BM * BK * 2;      // one weight tile: 16 KB
constexpr int NSTB = 5;                     // weight stages of the ring in this mode
constexpr int B_INPUT_BYTES = 49152;        // shared memory for one pass's input rows
constexpr int B_TMEM_COLS = 512;            // tensor-memory columns of the accumulators
static_assert(STAGE_BYTES == 2 * BOX_BYTES, "a weight stage holds two tiles");

// Geometry of a contraction of batch width BW.
template <int BW>
struct BGeo {
  static_assert(BW == 8 || BW == 16, "batch widths of whole 8-row swizzle atoms");
  static constexpr int BN = 2 * BW;                          // MMA N: hi columns, then lo columns
  static constexpr int KBLOCK_BYTES = BN * BK * 2;           // the hi and lo rows of one K block
  static constexpr int MAX_KBLOCKS = B_INPUT_BYTES / KBLOCK_BYTES;  // longest reduction segment of a pass
  static constexpr int NSLOT = B_TMEM_COLS / (2 * BN);       // accumulator slots of 2 BN columns
};
constexpr int NSLOT_MAX = BGeo<8>::NSLOT;
__host__ __device__ constexpr int batch_width(int R) { return R > 8 ? 16 : 8; }
__host__ __device__ constexpr int b_kblock_bytes(int bw) { return 4 * bw * BK; }
__host__ __device__ constexpr int b_max_kblocks(int bw) { return B_INPUT_BYTES / b_kblock_bytes(bw); }
__host__ __device__ constexpr int b_nslot(int bw) { return B_TMEM_COLS / (4 * bw); }
static_assert(b_kblock_bytes(8) == BGeo<8>::KBLOCK_BYTES && b_kblock_bytes(16) == BGeo<16>::KBLOCK_BYTES &&
                  b_max_kblocks(16) == BGeo<16>::MAX_KBLOCKS && b_nslot(16) == BGeo<16>::NSLOT,
              "host and device geometry agree");
static_assert(MAX_BATCH == MPK_MAX_BATCH && MAX_PREFILL == MPK_MAX_PREFILL && BM == MPK_BATCH_BM &&
                  BGeo<8>::MAX_KBLOCKS * BK == MPK_BATCH_MAX_PASS_K && BGeo<8>::NSLOT == MPK_BATCH_SLOTS &&
                  BGeo<16>::MAX_KBLOCKS * BK == MPK_BATCH_WIDE_MAX_PASS_K &&
                  BGeo<16>::NSLOT == MPK_BATCH_WIDE_SLOTS,
              "the header states the batched geometry");

enum TaskKind : int32_t {
  TK_EMBED = 1,
  TK_NORM_GEMV = 2,
  TK_ATTN = 3,
  TK_GEMV_RESID = 4,
  TK_NORM_GEMV_SILU = 5,
  TK_NORM_GEMV_ARGMAX = 6,
  TK_QKV_ATTN = 7,
};

// One operation of the compiled graph (device resident, read-only in the kernel).
struct OpDesc {
  int32_t kind;
  int32_t ntasks;          // tasks per iteration
  int32_t nwarps;          // consumer warps the task computes with (block_dim / 32)
  int32_t N;               // output rows of the GEMV (gate/up: I); embed: H
  int32_t K;               // reduction length
  int32_t rps;             // weight rows per stage (per matrix)
  int32_t nseg;            // number of stacked weight matrices (RMSNORM_LINEAR)
  int32_t seg_row0[MAX_SEG + 1];  // segment offsets within one group's rows
  int32_t groups;          // row groups (QKV+attention: kv heads; else 1); N = rows per group
  int32_t grp_rows[MAX_SEG];      // rows of segment s per group (matrix row = g * grp_rows + local)
  uint32_t* grp_cnt;       // QKV+attention: finished tasks per (request, group)
  int32_t ksplit;          // RESID: reduction split into ksplit segments of kseg (1: no split)
  int32_t kseg;
  uint64_t* kpart;         // RESID split: tagged partial sums [ksplit][N]
  uint32_t* blk_cnt;       // RESID split: finished segment tasks per row block
  const uint16_t* W[MAX_SEG];   // bf16 weights [rows, K]
  uint64_t* y[MAX_SEG];         // tagged outputs of RMSNORM_LINEAR
  const uint16_t* W_up;         // SILU: up matrix (W[0] = gate)
  const uint64_t* x;            // tagged input (norm ops) / residual (RESID)
  const uint64_t* a_in;         // tagged input of RESID
  const uint16_t* norm_w;       // bf16 [K]
  uint64_t* x_out;              // RESID: residual updated in place; EMBED: x (tagged)
  uint64_t* a_out;              // SILU / ATTN output (tagged)
  float eps;
  int32_t capture_slot;
  // attention
  int32_t layer, L, Hq, Hkv, d, G, C, S;
  const uint64_t* q;            // tagged
  const uint64_t* k;
  const uint64_t* v;
  const uint16_t* qn_w;
  const uint16_t* kn_w;
  uint16_t* kc;
  uint16_t* vc;
  // split-K operation: tensor maps of the caches viewed as [rows, d] bf16
  // (rows = L*R*Hkv*S, paged: L*npages*Hkv*page), boxes of 64 elements x
  // (STAGE_BYTES / (4 d)) rows, 128-byte swizzle
  const void* tmap_kc;
  const void* tmap_vc;
  // paged caches (split-K operation): page > 0 positions per page; the caches
  // are [L][npages][Hkv][page][d] and position p of request q lives in page
  // kv_pages[q * max_pages + p / page] at row p % page
  const int32_t* kv_pages;
  int32_t page, npages, max_pages;
  float* part;                  // [R][Hq][C][d + 2]
  uint64_t* gpart;              // group mode: tagged chunk partials [Hkv][C][G][d + 2]
  int32_t group_sync;           // fused op: every task of a group attends to a chunk (tasks <= workers)
  uint32_t* merge_cnt;          // [R][Hkv]
  const float2* rope;           // [S][d/2] (cos, sin)
  // embed / LM head
  const uint16_t* table;        // EMBED: embedding table [V][H]
  unsigned long long* keys;     // ARGMAX: per-request packed (value, index) maxima
  uint32_t* arrive;             // ARGMAX: arrival counter
  int64_t* pred;                // ARGMAX: optional [R][S]
  // versions: the tag of a value written by op w in iteration n is n * nops + w + 1
  int32_t self;                 // this op's index (the writer of its outputs)
  int32_t x_writer;             // op that last wrote the x this op reads (-1: none)
  int32_t a_writer;             // op that wrote a_in (RESID) or q/k/v (attention)
  int32_t tagged;               // 1: inputs are waited for through their tags; 0: through dep_event
  int32_t dynamic;              // 1: workers claim this op's tasks from a shared counter
  uint32_t tag_skew;            // added to every expected input tag (0; fault injection for tests)
  // events
  int32_t dep_event;            // event this op waits on
  int32_t dep_trigger;          // increments of dep_event per iteration
  int32_t dep_iter_offset;      // wait for (iter + offset) * trigger
  int32_t out_event;            // event this op signals
  int32_t out_trigger;          // increments of out_event per iteration
  int32_t signal_per_task;      // 1: every task signals; 0: merges / finisher signal
  // tensor-core path (batched)
  int32_t batched;              // 1: the projection runs as tcgen05 MMAs over the batch
  int32_t nb;                   // row blocks of BM rows (gate/up: of one matrix)
  int32_t nkb;                  // K blocks of BK elements
  int32_t bsplit;               // reduction segments (grid_dim.y)
  int32_t ntb;                  // tasks per segment (grid_dim.x), each owning a run of row blocks
  const void* tmap[MAX_SEG];    // tensor maps of W[s] (device memory, 64-byte aligned)
  const void* tmap_up;          // SILU: tensor map of the up matrix
  float* bpart;                 // bsplit > 1: partial sums [bsplit][N][BW] (gate/up: [..][2 BW])
  // per-block sums of squares of x (batched graphs): EMBED and RESID publish
  // them for every BM-row block of the x they write, tagged [blocks][R]; the
  // RMSNorm operations read them instead of the whole of x
  uint64_t* xss_out;
  const uint64_t* xss_in;
  int32_t xss_blocks;
  // published input rows (batched graphs): the writer of a projection's input
  // also stores it as bf16 hi/lo in the swizzled layout of the shared-memory
  // input buffer ([K/64 blocks][2 x BW rows][64], 4 BW * 64 bytes per block; rows past R
  // zero) and the reader copies its K blocks with one bulk copy.  Writers of x
  // (EMBED, RESID) store x * w_norm of the next RMSNorm operation (xb_w) and
  // release the rows with the block's sums of squares; the reader applies the
  // RMS factor to the products.  Writers of a projection's plain input (the
  // attention's merge, the gate/up epilogue; xb_w null) release them with tagged
  // flags: flag r * xf_rstride + k / xf_grp covers element k of request r.
  uint16_t* xb_out;
  const uint16_t* xb_w;
  const uint16_t* xb_in;
  uint64_t* xf_out;
  const uint64_t* xf_in;
  int32_t xf_grp;
  int32_t xf_rstride;
};

struct Status {
  int32_t code;      // 0 ok, else negative mpk_error
  int32_t where;     // 1 worker dep, 2 producer queue, 3 producer ring, 4 consumer fifo, 5 scheduler gate, 6 scheduler space, 7 start,
                     // 8 token check, 9 task dispatch, 10 iteration boundary, 11 tagged input, 12 KV page check
  int32_t op, task, worker, iter;
  uint32_t observed, expected;
};

constexpr int MAX_REQUESTS = 64;
struct Control {
  uint32_t ready;
  uint32_t n_iter;
  uint32_t pad[30];
  // per request, read at the start of a run: step[r] (-1: inactive) and the
  // last position it may reach, min(step_end[r], S - 1).  While a request is
  // active its step advances by exactly one per iteration, so in iteration n
  // it is step0[r] + n.  A prefill graph serves its requests one after
  // another, R positions per iteration; cum[q] is the number of iterations
  // before request q's first (cum[Rq]: all of the run's).
  int32_t step0[MAX_REQUESTS];
  int32_t stop[MAX_REQUESTS];
  uint32_t cum[MAX_REQUESTS + 1];
};

struct Graph {
  const OpDesc* ops;
  int32_t nops;
  int32_t op_by_op;                 // 1: every operation is its own launch (mpk_run_op_by_op)
  int32_t batched;                  // 1: projections run on the tensor-core path (R >= 2)
  int32_t bw;                       // batched: batch width of the contractions (8 or 16)
  int32_t split_attn;               // 1: the graph has split-K attention operations
  int32_t prefill;                  // 1: the R columns are R consecutive positions of one request
  int32_t Rq;                       // requests of tokens, step, pred and the KV cache (without prefill: R)
  int32_t R, S, V, H, L;
  int32_t num_workers, num_sched;   // scheduler warps
  int32_t sched_ctas;
  int32_t lookahead;
  uint32_t prefetch_bytes;          // L2 prefetch distance per worker (0 = off)
  uint32_t* events;                 // [nops] (one 128-byte line each)
  uint32_t* claims;                 // [CLAIM_SLOTS][nops] task-claim counters (one line each)
  unsigned long long* queue;        // [num_workers][QUEUE_CAP]
  uint32_t* q_head;                 // [num_workers] (one line each)
  uint32_t* q_tail;
  int32_t* step;
  int64_t* tokens;
  const int32_t* step_end;
  Control* ctl;
  Status* status;
  volatile int32_t* abort_flag;     // host-mapped
  uint64_t timeout_ns;
  int32_t capture_iter;
  float* cap_logits;
  float* cap_hidden;
  int32_t profiling;
  int32_t max_timeline;
  unsigned long long* timeline;     // [max_timeline][TIMELINE_FIELDS]
  uint32_t* timeline_n;
};

// entry, worker, popped, dependency met, end, prologue done, first stage ready,
// first stage issued, time spent waiting for weight stages, last stage ready,
// rows done
constexpr int TIMELINE_FIELDS = MPK_TIMELINE_FIELDS;
constexpr int EVENT_STRIDE = 32;    // uint32 per event / queue counter (128 bytes)
constexpr unsigned long long QUEUE_TERMINATE = ~0ull;
// Task field of a queue entry that stands for "claim tasks of this dynamic
// operation until none is left" (one such entry per worker).
constexpr uint32_t TASK_CLAIM = 0xFFFFu;
constexpr int CLAIM_SLOTS = 4;  // claim counters per op, used by iteration n % CLAIM_SLOTS

__host__ __device__ inline unsigned long long pack_entry(uint32_t iter, uint32_t op, uint32_t task) {
  return ((unsigned long long)iter << 32) | ((unsigned long long)op << 16) | (unsigned long long)task;
}

}  // namespace mpk
