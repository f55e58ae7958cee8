// Host side of the C ABI declared in include/mpk.h: tensor registry, graph
// compiler (validation, task split, event assignment, workspace layout) and
// the launch of the persistent kernel.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "mpk.h"
#include "mpk_internal.h"

namespace mpk {
size_t kernel_smem_bytes();
cudaError_t prepare_kernels();
cudaError_t max_blocks_per_sm(int* n);
cudaError_t launch_persistent(const Graph& g, int grid, cudaStream_t stream);
cudaError_t launch_op(const Graph& g, int op, int ntasks, uint32_t iter, bool cooperative, cudaStream_t stream);
}  // namespace mpk

using namespace mpk;

namespace {

struct Tensor {
  void* ptr = nullptr;
  mpk_dtype dtype = MPK_BF16;
  std::vector<int64_t> dims;
  bool owned = false;
};

size_t dtype_size(mpk_dtype t) {
  switch (t) {
    case MPK_BF16: return 2;
    case MPK_FP32: return 4;
    case MPK_INT32: return 4;
    case MPK_INT64: return 8;
    case MPK_FP32T: return 8;
  }
  return 0;
}

const char* dtype_name(mpk_dtype t) {
  switch (t) {
    case MPK_BF16: return "bf16";
    case MPK_FP32: return "fp32";
    case MPK_INT32: return "int32";
    case MPK_INT64: return "int64";
    case MPK_FP32T: return "fp32t";
  }
  return "?";
}

std::string g_create_error;

}  // namespace

struct mpk_ctx {
  int device = 0, sms = 0;
  int num_workers = 0, num_local = 0, num_remote = 0;
  std::map<std::string, Tensor> tensors;
  bool compiled = false;
  std::vector<OpDesc> ops;
  OpDesc* ops_dev = nullptr;
  Graph graph{};
  std::vector<void*> allocs;      // library-owned device memory
  void* sync_block = nullptr;     // per-run zeroed state
  size_t sync_bytes = 0;
  int32_t* abort_host = nullptr;  // mapped
  Status* status_dev = nullptr;
  int32_t R = 0, S_cache = 0, V = 0, H = 0, L = 0;
  int32_t pred_S = 0;
  int32_t prefill = 0;  // columns of a prefill graph (0: one position per request per iteration)
  int32_t Rq = 0;       // requests of tokens, step, pred and the KV cache (without prefill: R)
  std::string err, warnings;
  std::vector<std::pair<void*, size_t>> zero_each_run;  // tagged activations: versions restart at every run
  int capture_iter = -1;
  float* cap_logits = nullptr;
  float* cap_hidden = nullptr;
  mpk_options opts{};
};

namespace {

int fail(mpk_ctx* c, int code, const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (c) c->err = buf;
  else g_create_error = buf;
  return code;
}

#define CUDA_OR_FAIL(ctx, call)                                                          \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess)                                                               \
      return fail(ctx, MPK_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));   \
  } while (0)

const Tensor* find(mpk_ctx* c, const char* name) {
  if (!name) return nullptr;
  auto it = c->tensors.find(name);
  return it == c->tensors.end() ? nullptr : &it->second;
}

std::string dims_str(const std::vector<int64_t>& d) {
  std::string s = "[";
  for (size_t i = 0; i < d.size(); ++i) s += (i ? "," : "") + std::to_string(d[i]);
  return s + "]";
}

// Fetch tensor `name`, check dtype and rank; fill *out.
int need(mpk_ctx* c, int li, const char* role, const char* name, mpk_dtype dt, int ndim, const Tensor** out) {
  if (!name) return fail(c, MPK_ERR_INVALID_ARG, "layer %d: %s name missing", li, role);
  const Tensor* t = find(c, name);
  if (!t) return fail(c, MPK_ERR_NOT_FOUND, "layer %d: %s tensor '%s' not registered", li, role, name);
  if (t->dtype != dt)
    return fail(c, MPK_ERR_DTYPE, "layer %d: %s '%s' is %s, expected %s", li, role, name, dtype_name(t->dtype),
                dtype_name(dt));
  if ((int)t->dims.size() != ndim)
    return fail(c, MPK_ERR_SHAPE, "layer %d: %s '%s' has shape %s, expected rank %d", li, role, name,
                dims_str(t->dims).c_str(), ndim);
  *out = t;
  return MPK_OK;
}

#define NEED(role, name, dt, nd, out)                       \
  do {                                                      \
    int rc_ = need(c, li, role, name, dt, nd, out);         \
    if (rc_ != MPK_OK) return rc_;                          \
  } while (0)

#define SHAPE_CHECK(cond, ...)                              \
  do {                                                      \
    if (!(cond)) return fail(c, MPK_ERR_SHAPE, __VA_ARGS__); \
  } while (0)

// GEMV geometry: rows per shared-memory stage (each consumer warp owns whole
// rows, so any K that is a multiple of 256 and fits the input buffer works).
int gemv_geometry(mpk_ctx* c, int li, OpDesc& o, bool two_mats, bool norm) {
  const int K = o.ksplit > 1 ? o.kseg : o.K;
  if (K % 256 != 0) return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: reduction length %d is not a multiple of 256", li, K);
  if (K > MAX_K) return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: reduction length %d exceeds %d", li, K, MAX_K);
  if (norm && K > MAX_NORM_K)
    return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: RMSNorm width %d exceeds %d", li, K, MAX_NORM_K);
  const int row_bytes = K * 2 * (two_mats ? 2 : 1);
  int rps = STAGE_BYTES / row_bytes;
  if (rps < 1) return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: one weight row (%d bytes) exceeds a stage", li, row_bytes);
  if (rps > MAX_RPS) rps = MAX_RPS;
  o.rps = rps;
  return MPK_OK;
}

// Tensor-core geometry of a projection over R >= 2 requests: row blocks of BM,
// K blocks of BK; grid_dim = (tasks per reduction segment, reduction segments,
// 1).  Task t computes segment t / gx for the run of row blocks
// [u nb / gx, (u+1) nb / gx), u = t mod gx, so gx <= nb.
int batched_geometry(mpk_ctx* c, int li, OpDesc& o, int R, const mpk_layer& Ly) {
  if (R > MAX_BATCH)
    return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: %d requests (the batched projections take at most %d)", li, R,
                MAX_BATCH);
  if (o.K % BK != 0)
    return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: reduction length %d is not a multiple of %d", li, o.K, BK);
  for (int s = 1; s < o.nseg; ++s)
    if (o.seg_row0[s] % BM != 0)
      return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: stacked matrix %d starts at row %d, not a multiple of %d", li, s,
                  o.seg_row0[s], BM);
  const int gx = Ly.grid_dim.x, gy = Ly.grid_dim.y > 0 ? Ly.grid_dim.y : 1,
            gz = Ly.grid_dim.z > 0 ? Ly.grid_dim.z : 1;
  o.batched = 1;
  o.nb = (o.N + BM - 1) / BM;
  o.nkb = o.K / BK;
  o.ntb = gx;
  o.bsplit = gy;
  if (gz != 1)
    return fail(c, MPK_ERR_SHAPE, "layer %d: a batched projection takes grid_dim = (row-block tasks, reduction "
                "segments, 1)", li);
  if (gx > o.nb)
    return fail(c, MPK_ERR_SHAPE, "layer %d: %d rows are %d blocks of %d: grid_dim.x = %d tasks per segment is more",
                li, o.N, o.nb, BM, gx);
  if (gy > o.nkb)
    return fail(c, MPK_ERR_SHAPE, "layer %d: grid_dim.y = %d segments for a reduction of %d blocks of %d", li, gy,
                o.nkb, BK);
  // a segment longer than the input buffer runs in passes, which keep every
  // row block of the task in its own tensor-memory accumulator slot
  const int bw = batch_width(R), max_kblocks = b_max_kblocks(bw), nslot = b_nslot(bw);
  const int longest = (o.nkb + gy - 1) / gy;
  const int most_blocks = (o.nb + gx - 1) / gx;
  if (longest > max_kblocks && most_blocks > nslot)
    return fail(c, MPK_ERR_SHAPE,
                "layer %d: tasks of %d row blocks over %d elements of the reduction: a task longer than %d elements "
                "takes at most %d row blocks (more tasks per segment, grid_dim.x, or more segments, grid_dim.y)",
                li, most_blocks, longest * BK, max_kblocks * BK, nslot);
  o.dynamic = 0;
  return MPK_OK;
}

// Tensor map of a bf16 [rows, K] row-major matrix for box_rows x BK tiles
// with 128-byte swizzle (the layout the MMA's shared-memory descriptors and the
// attention's matrix loads expect).
int make_weight_map(mpk_ctx* c, int li, CUtensorMap* m, const void* ptr, int64_t rows, int64_t K,
                    int box_rows = BM) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return fail(c, MPK_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(c, MPK_ERR_CUDA, "layer %d: tensor map of a [%lld, %lld] weight failed (CUresult %d)", li,
                (long long)rows, (long long)K, (int)r);
  return MPK_OK;
}

int check_grid(mpk_ctx* c, int li, const mpk_layer& Ly, int ntasks, int rows) {
  if (ntasks < 1 || ntasks > 65535)
    return fail(c, MPK_ERR_INVALID_ARG, "layer %d: grid_dim gives %d tasks (1..65535)", li, ntasks);
  if (rows > 0 && ntasks > rows)
    return fail(c, MPK_ERR_SHAPE, "layer %d: %d tasks for %d rows (at most one task per row)", li, ntasks, rows);
  if (ntasks % c->num_workers != 0) {
    char b[256];
    snprintf(b, sizeof b, "layer %d: %d tasks is not a multiple of num_workers=%d (some workers idle in this phase)\n",
             li, ntasks, c->num_workers);
    c->warnings += b;
  }
  (void)Ly;
  return MPK_OK;
}

template <typename T>
int alloc(mpk_ctx* c, T** p, size_t bytes) {
  void* q = nullptr;
  CUDA_OR_FAIL(c, cudaMalloc(&q, bytes ? bytes : 16));
  CUDA_OR_FAIL(c, cudaMemset(q, 0, bytes ? bytes : 16));
  c->allocs.push_back(q);
  *p = reinterpret_cast<T*>(q);
  return MPK_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int mpk_abi_version(void) { return MPK_ABI_VERSION; }
int mpk_worker_threads(void) { return CONSUMER_THREADS; }

int mpk_device_sm_count(void) {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MPK_ERR_CUDA;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MPK_ERR_CUDA;
  return n;
}

static int validate_split(int sms, int num_workers, int num_local_schedulers, int num_remote_schedulers) {
  if (num_workers < 1 || num_local_schedulers < 0 || num_remote_schedulers < 0)
    return fail(nullptr, MPK_ERR_INVALID_ARG, "counts must be positive (workers %d, local %d, remote %d)", num_workers,
                num_local_schedulers, num_remote_schedulers);
  const int sched = num_local_schedulers + num_remote_schedulers;
  if (sched % 4 != 0)
    return fail(nullptr, MPK_ERR_SM_FORMULA,
                "num_local_schedulers + num_remote_schedulers = %d is not a multiple of 4", sched);
  if (num_workers + sched / 4 != sms)
    return fail(nullptr, MPK_ERR_SM_FORMULA,
                "num_workers + (num_local_schedulers + num_remote_schedulers) / 4 = %d + %d = %d, but the GPU has %d SMs",
                num_workers, sched / 4, num_workers + sched / 4, sms);
  if (num_remote_schedulers != 0)
    return fail(nullptr, MPK_ERR_UNSUPPORTED, "remote schedulers serve other GPUs; this build runs on one GPU");
  if (num_local_schedulers == 0)
    return fail(nullptr, MPK_ERR_INVALID_ARG, "at least one group of 4 local schedulers is required");
  return MPK_OK;
}

int mpk_validate_split(int sm_count, int num_workers, int num_local_schedulers, int num_remote_schedulers) {
  return validate_split(sm_count, num_workers, num_local_schedulers, num_remote_schedulers);
}

int mpk_create(int num_workers, int num_local_schedulers, int num_remote_schedulers, mpk_ctx** out) {
  if (!out) return fail(nullptr, MPK_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  int dev = 0, sms = 0, major = 0, minor = 0, coop = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(nullptr, MPK_ERR_CUDA, "no CUDA device");
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
  const int rc_split = validate_split(sms, num_workers, num_local_schedulers, num_remote_schedulers);
  if (rc_split != MPK_OK) return rc_split;
  if (major != 10 || minor != 0)
    return fail(nullptr, MPK_ERR_UNSUPPORTED, "device is sm_%d%d; this library is built for sm_100a", major, minor);
  if (!coop) return fail(nullptr, MPK_ERR_UNSUPPORTED, "device lacks cooperative launch");
  cudaError_t e = prepare_kernels();
  if (e != cudaSuccess) return fail(nullptr, MPK_ERR_CUDA, "kernel setup failed: %s", cudaGetErrorString(e));
  int per_sm = 0;
  e = max_blocks_per_sm(&per_sm);
  if (e != cudaSuccess || per_sm < 1)
    return fail(nullptr, MPK_ERR_UNSUPPORTED, "persistent kernel cannot be resident (%d blocks/SM): %s", per_sm,
                cudaGetErrorString(e));
  mpk_ctx* c = new mpk_ctx();
  c->device = dev;
  c->sms = sms;
  c->num_workers = num_workers;
  c->num_local = num_local_schedulers;
  c->num_remote = num_remote_schedulers;
  if (cudaHostAlloc(reinterpret_cast<void**>(&c->abort_host), 64, cudaHostAllocMapped) != cudaSuccess) {
    delete c;
    return fail(nullptr, MPK_ERR_CUDA, "cudaHostAlloc of the abort flag failed");
  }
  *c->abort_host = 0;
  *out = c;
  return MPK_OK;
}

static int register_tensor(mpk_ctx* c, const char* name, void* ptr, mpk_dtype dtype, int ndim, const int64_t* dims,
                           bool owned) {
  if (!name || !*name) return fail(c, MPK_ERR_INVALID_ARG, "tensor name is empty");
  if (c->compiled) return fail(c, MPK_ERR_STATE, "tensors cannot be added after compile");
  if (ndim < 1 || ndim > 5 || !dims) return fail(c, MPK_ERR_INVALID_ARG, "'%s': rank must be 1..5", name);
  if ((int)dtype < 0 || (int)dtype > 4) return fail(c, MPK_ERR_INVALID_ARG, "'%s': unknown dtype %d", name, (int)dtype);
  if (c->tensors.count(name)) return fail(c, MPK_ERR_INVALID_ARG, "tensor '%s' already registered", name);
  Tensor t;
  for (int i = 0; i < ndim; ++i) {
    if (dims[i] < 1) return fail(c, MPK_ERR_INVALID_ARG, "'%s': extent %lld < 1", name, (long long)dims[i]);
    t.dims.push_back(dims[i]);
  }
  if (!owned) {
    if (!ptr) return fail(c, MPK_ERR_INVALID_ARG, "'%s': device pointer is NULL", name);
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0)
      return fail(c, MPK_ERR_INVALID_ARG, "'%s': pointer is not 16-byte aligned", name);
  }
  t.ptr = ptr;
  t.dtype = dtype;
  t.owned = owned;
  c->tensors[name] = t;
  return MPK_OK;
}

int mpk_attach_input(mpk_ctx* c, const char* name, void* dev_ptr, mpk_dtype dtype, int ndim, const int64_t* dims) {
  if (!c) return MPK_ERR_INVALID_ARG;
  return register_tensor(c, name, dev_ptr, dtype, ndim, dims, false);
}

int mpk_new_tensor(mpk_ctx* c, const char* name, mpk_dtype dtype, int ndim, const int64_t* dims, mpk_io io,
                   void** dev_ptr_out) {
  if (!c) return MPK_ERR_INVALID_ARG;
  if (io == MPK_IO_NVSHMEM)
    return fail(c, MPK_ERR_UNSUPPORTED, "'%s': nvshmem_tensor is for remote GPU access; this build runs on one GPU",
                name ? name : "");
  if (io != MPK_IO_CUDA) return fail(c, MPK_ERR_INVALID_ARG, "unknown io category %d", (int)io);
  if ((int)dtype < 0 || (int)dtype > 4) return fail(c, MPK_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (ndim < 1 || ndim > 5 || !dims) return fail(c, MPK_ERR_INVALID_ARG, "rank must be 1..5");
  int64_t n = 1;
  for (int i = 0; i < ndim; ++i) {
    if (dims[i] < 1) return fail(c, MPK_ERR_INVALID_ARG, "extent < 1");
    n *= dims[i];
  }
  if (name && c->tensors.count(name)) return fail(c, MPK_ERR_INVALID_ARG, "tensor '%s' already registered", name);
  if (c->compiled) return fail(c, MPK_ERR_STATE, "tensors cannot be added after compile");
  void* p = nullptr;
  int rc = alloc(c, &p, (size_t)n * dtype_size(dtype));
  if (rc != MPK_OK) return rc;
  rc = register_tensor(c, name, p, dtype, ndim, dims, true);
  if (rc != MPK_OK) return rc;
  if (dev_ptr_out) *dev_ptr_out = p;
  return MPK_OK;
}

void* mpk_tensor_ptr(mpk_ctx* c, const char* name) {
  if (!c) return nullptr;
  const Tensor* t = find(c, name);
  return t ? t->ptr : nullptr;
}

const char* mpk_warnings(mpk_ctx* c) { return c ? c->warnings.c_str() : ""; }

int mpk_compile(mpk_ctx* c, const mpk_layer* layers, int n_layers, const mpk_options* opts) {
  if (!c) return MPK_ERR_INVALID_ARG;
  if (c->compiled) return fail(c, MPK_ERR_STATE, "already compiled");
  if (!layers || n_layers < 1) return fail(c, MPK_ERR_INVALID_ARG, "no layers");
  if (n_layers > 65535) return fail(c, MPK_ERR_INVALID_ARG, "too many layers");
  c->warnings.clear();
  mpk_options o{};
  if (opts) o = *opts;
  if (o.sched_lookahead <= 0) o.sched_lookahead = 4;
  if (o.timeout_s <= 0) o.timeout_s = 2.0;
  if (o.max_timeline <= 0) o.max_timeline = 1 << 20;
  if (o.prefetch_kb == 0) o.prefetch_kb = -1;
  c->opts = o;
  // a prefill graph: its R columns are consecutive positions of one request
  // of the KV cache, which may hold any number of requests (Rq)
  const int PF = o.prefill_tokens > 1 ? o.prefill_tokens : 0;
  int Rq = -1;
  // paged KV caches: [L, pages, Hkv, PG, d] and the page table "kv_pages"
  // [requests, max_pages] (int32)
  const int PG = o.kv_page_size > 0 ? o.kv_page_size : 0;
  const Tensor* kvp = nullptr;
  if (PG) {
    if (PG % 128 != 0)
      return fail(c, MPK_ERR_INVALID_ARG, "kv_page_size %d is not a multiple of 128", PG);
    int rc_ = need(c, -1, "page table", "kv_pages", MPK_INT32, 2, &kvp);
    if (rc_ != MPK_OK) return rc_;
    if (kvp->dims[0] < 1 || kvp->dims[1] < 1 || (int64_t)kvp->dims[1] * PG >= ((int64_t)1 << 31))
      return fail(c, MPK_ERR_SHAPE, "kv_pages %s", dims_str(kvp->dims).c_str());
  }

  std::vector<OpDesc> ops(n_layers);
  int R = -1, H = -1, V = -1, L = -1, S = -1, pred_rows = -1;
  // attention workspace sizing
  size_t part_floats = 0, merge_u32 = 0, kpart_floats = 0, blk_u32 = 0, gpart_words = 0;
  std::vector<std::pair<int, size_t>> merge_off(n_layers, {0, 0});
  struct RopeKey { float theta; int d; int S; };
  std::vector<RopeKey> rope_keys;
  std::vector<int> rope_of(n_layers, -1);
  int n_argmax = 0;

  for (int li = 0; li < n_layers; ++li) {
    const mpk_layer& Ly = layers[li];
    OpDesc& op = ops[li];
    memset(&op, 0, sizeof(op));
    op.groups = 1;
    op.capture_slot = Ly.capture_slot;
    op.eps = Ly.eps > 0 ? Ly.eps : 1e-6f;
    const int64_t ntasks64 = (int64_t)Ly.grid_dim.x * (Ly.grid_dim.y > 0 ? Ly.grid_dim.y : 1) *
                             (Ly.grid_dim.z > 0 ? Ly.grid_dim.z : 1);
    if (Ly.grid_dim.x < 1 || ntasks64 > 65535)
      return fail(c, MPK_ERR_INVALID_ARG, "layer %d: grid_dim must give 1..65535 tasks", li);
    const int ntasks = (int)ntasks64;
    const int64_t threads = (int64_t)(Ly.block_dim.x > 0 ? Ly.block_dim.x : CONSUMER_THREADS) *
                            (Ly.block_dim.y > 0 ? Ly.block_dim.y : 1) * (Ly.block_dim.z > 0 ? Ly.block_dim.z : 1);
    if (threads < 32 || threads > CONSUMER_THREADS || threads % 32 != 0)
      return fail(c, MPK_ERR_INVALID_ARG, "layer %d: block_dim gives %lld threads (a multiple of 32, at most %d)", li,
                  (long long)threads, CONSUMER_THREADS);
    op.nwarps = (int)(threads / 32);
    op.ntasks = ntasks;
    const Tensor *x, *w0, *w1, *w2, *out;
    switch (Ly.op) {
      case MPK_OP_EMBED: {
        op.kind = TK_EMBED;
        NEED("weights[0] (embedding)", Ly.weights[0], MPK_BF16, 2, &w0);
        NEED("outputs[0] (x)", Ly.outputs[0], MPK_FP32T, 2, &out);
        SHAPE_CHECK(out->dims[1] == w0->dims[1], "layer %d: x width %lld != embedding width %lld", li,
                    (long long)out->dims[1], (long long)w0->dims[1]);
        SHAPE_CHECK(out->dims[1] % 8 == 0, "layer %d: hidden size must be a multiple of 8", li);
        if (R < 0) R = (int)out->dims[0];
        SHAPE_CHECK(out->dims[0] == R, "layer %d: request count mismatch", li);
        SHAPE_CHECK(ntasks == R, "layer %d: EMBED needs grid_dim = number of requests (%d)", li, R);
        op.table = (const uint16_t*)w0->ptr;
        op.x_out = (uint64_t*)out->ptr;
        op.N = (int)out->dims[1];
        if (V < 0) V = (int)w0->dims[0];
        if (H < 0) H = op.N;
        op.signal_per_task = 1;
        op.out_trigger = ntasks;
        break;
      }
      case MPK_OP_RMSNORM_LINEAR:
      case MPK_OP_LINEAR_RESIDUAL:
      case MPK_OP_RMSNORM_LINEAR_SILU_MUL:
      case MPK_OP_RMSNORM_LMHEAD_ARGMAX: {
        const bool resid = Ly.op == MPK_OP_LINEAR_RESIDUAL;
        const bool silu = Ly.op == MPK_OP_RMSNORM_LINEAR_SILU_MUL;
        const bool lmh = Ly.op == MPK_OP_RMSNORM_LMHEAD_ARGMAX;
        op.kind = resid ? TK_GEMV_RESID : silu ? TK_NORM_GEMV_SILU : lmh ? TK_NORM_GEMV_ARGMAX : TK_NORM_GEMV;
        if (resid) {
          NEED("inputs[0] (a)", Ly.inputs[0], MPK_FP32T, 2, &x);
          op.a_in = (const uint64_t*)x->ptr;
          op.K = (int)x->dims[1];
          NEED("weights[0] (W)", Ly.weights[0], MPK_BF16, 2, &w0);
          NEED("outputs[0] (x)", Ly.outputs[0], MPK_FP32T, 2, &out);
          SHAPE_CHECK(w0->dims[1] == op.K, "layer %d: W is %s but input has %d features", li,
                      dims_str(w0->dims).c_str(), op.K);
          SHAPE_CHECK(out->dims[1] == w0->dims[0] && out->dims[0] == x->dims[0],
                      "layer %d: residual %s does not match W %s", li, dims_str(out->dims).c_str(),
                      dims_str(w0->dims).c_str());
          op.N = (int)w0->dims[0];
          op.W[0] = (const uint16_t*)w0->ptr;
          op.nseg = 1;
          op.seg_row0[0] = 0;
          op.seg_row0[1] = op.N;
          op.x_out = (uint64_t*)out->ptr;
          op.x = (const uint64_t*)out->ptr;
          if (op.K > MAX_K && x->dims[0] < 2) {
            // One request: split the reduction into the fewest segments that
            // fit the input buffer (several requests split it on their own
            // terms, see batched_geometry).
            int ks = (op.K + MAX_K - 1) / MAX_K;
            while (ks <= op.K / 256 && (op.K % ks != 0 || (op.K / ks) % 256 != 0)) ++ks;
            if (ks > op.K / 256 || ks > MAX_KSPLIT)
              return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: reduction length %d cannot be split into at most %d "
                          "segments", li, op.K, MAX_KSPLIT);
            if (ntasks % ks != 0)
              return fail(c, MPK_ERR_SHAPE,
                          "layer %d: reduction length %d is split into %d segments: grid_dim must give a multiple "
                          "of %d tasks (got %d)", li, op.K, ks, ks, ntasks);
            op.ksplit = ks;
            op.kseg = op.K / ks;
            kpart_floats = std::max(kpart_floats, (size_t)ks * op.N);
            blk_u32 = std::max(blk_u32, (size_t)(ntasks / ks));
          }
        } else {
          NEED("inputs[0] (x)", Ly.inputs[0], MPK_FP32T, 2, &x);
          op.x = (const uint64_t*)x->ptr;
          op.K = (int)x->dims[1];
          NEED("weights[0] (norm)", Ly.weights[0], MPK_BF16, 1, &w0);
          SHAPE_CHECK(w0->dims[0] == op.K, "layer %d: norm weight %s, input width %d", li, dims_str(w0->dims).c_str(),
                      op.K);
          op.norm_w = (const uint16_t*)w0->ptr;
          if (silu) {
            NEED("weights[1] (gate)", Ly.weights[1], MPK_BF16, 2, &w1);
            NEED("weights[2] (up)", Ly.weights[2], MPK_BF16, 2, &w2);
            NEED("outputs[0] (a)", Ly.outputs[0], MPK_FP32T, 2, &out);
            SHAPE_CHECK(w1->dims == w2->dims && w1->dims[1] == op.K, "layer %d: gate %s / up %s vs K=%d", li,
                        dims_str(w1->dims).c_str(), dims_str(w2->dims).c_str(), op.K);
            SHAPE_CHECK(out->dims[1] == w1->dims[0] && out->dims[0] == x->dims[0], "layer %d: output %s", li,
                        dims_str(out->dims).c_str());
            op.N = (int)w1->dims[0];
            op.W[0] = (const uint16_t*)w1->ptr;
            op.W_up = (const uint16_t*)w2->ptr;
            op.nseg = 1;
            op.seg_row0[0] = 0;
            op.seg_row0[1] = op.N;
            op.a_out = (uint64_t*)out->ptr;
          } else if (lmh) {
            NEED("weights[1] (lm head)", Ly.weights[1], MPK_BF16, 2, &w1);
            SHAPE_CHECK(w1->dims[1] == op.K, "layer %d: LM head %s vs K=%d", li, dims_str(w1->dims).c_str(), op.K);
            op.N = (int)w1->dims[0];
            op.W[0] = (const uint16_t*)w1->ptr;
            op.nseg = 1;
            op.seg_row0[0] = 0;
            op.seg_row0[1] = op.N;
            if (Ly.outputs[0]) {
              NEED("outputs[0] (pred)", Ly.outputs[0], MPK_INT64, 2, &out);
              op.pred = (int64_t*)out->ptr;
              if (S < 0) S = (int)out->dims[1];
              pred_rows = (int)out->dims[0];
            }
            if (V < 0) V = op.N;
            SHAPE_CHECK(op.N == V, "layer %d: LM head rows %d != vocabulary %d", li, op.N, V);
            if (li != n_layers - 1)
              return fail(c, MPK_ERR_INVALID_ARG, "layer %d: the LM-head/argmax operation must be last", li);
            ++n_argmax;
          } else {
            op.nseg = 0;
            int rows = 0;
            for (int s = 0; s < MAX_SEG; ++s) {
              if (!Ly.weights[1 + s]) break;
              const Tensor *ws, *ys;
              NEED("weights[1+i] (linear)", Ly.weights[1 + s], MPK_BF16, 2, &ws);
              if (!Ly.outputs[s]) return fail(c, MPK_ERR_INVALID_ARG, "layer %d: outputs[%d] missing", li, s);
              NEED("outputs[i]", Ly.outputs[s], MPK_FP32T, 2, &ys);
              SHAPE_CHECK(ws->dims[1] == op.K && ys->dims[1] == ws->dims[0] && ys->dims[0] == x->dims[0],
                          "layer %d: linear %d W %s, y %s, K=%d", li, s, dims_str(ws->dims).c_str(),
                          dims_str(ys->dims).c_str(), op.K);
              op.W[s] = (const uint16_t*)ws->ptr;
              op.y[s] = (uint64_t*)ys->ptr;
              op.seg_row0[s] = rows;
              rows += (int)ws->dims[0];
              op.nseg = s + 1;
            }
            if (op.nseg == 0) return fail(c, MPK_ERR_INVALID_ARG, "layer %d: no linear weight", li);
            op.seg_row0[op.nseg] = rows;
            for (int s = op.nseg + 1; s <= MAX_SEG; ++s) op.seg_row0[s] = rows;
            for (int s = 0; s < op.nseg; ++s) op.grp_rows[s] = op.seg_row0[s + 1] - op.seg_row0[s];
            op.N = rows;
          }
        }
        if (R < 0) R = (int)x->dims[0];
        SHAPE_CHECK(x->dims[0] == R, "layer %d: %lld requests, graph has %d", li, (long long)x->dims[0], R);
        if (R >= 2) {
          // several requests: the projection is a dense contraction on the tensor cores
          op.ksplit = 0;
          op.kseg = 0;
          int rc = batched_geometry(c, li, op, R, Ly);
          if (rc != MPK_OK) return rc;
          rc = check_grid(c, li, Ly, ntasks, 0);
          if (rc != MPK_OK) return rc;
        } else {
          int rc = gemv_geometry(c, li, op, silu, !resid);
          if (rc != MPK_OK) return rc;
          rc = check_grid(c, li, Ly, ntasks, op.N * (op.ksplit > 1 ? op.ksplit : 1));
          if (rc != MPK_OK) return rc;
        }
        op.signal_per_task = lmh ? 0 : 1;
        op.out_trigger = lmh ? 1 : ntasks;
        if (resid && H < 0) H = op.N;
        break;
      }
      case MPK_OP_ATTENTION: {
        op.kind = TK_ATTN;
        const Tensor *q, *k, *v, *qn, *kn, *kc, *vc, *o;
        NEED("inputs[0] (q)", Ly.inputs[0], MPK_FP32T, 2, &q);
        NEED("inputs[1] (k)", Ly.inputs[1], MPK_FP32T, 2, &k);
        NEED("inputs[2] (v)", Ly.inputs[2], MPK_FP32T, 2, &v);
        NEED("weights[0] (q_norm)", Ly.weights[0], MPK_BF16, 1, &qn);
        NEED("weights[1] (k_norm)", Ly.weights[1], MPK_BF16, 1, &kn);
        NEED("weights[2] (k_cache)", Ly.weights[2], MPK_BF16, 5, &kc);
        NEED("weights[3] (v_cache)", Ly.weights[3], MPK_BF16, 5, &vc);
        NEED("outputs[0] (o)", Ly.outputs[0], MPK_FP32T, 2, &o);
        SHAPE_CHECK(kc->dims == vc->dims, "layer %d: k/v caches differ", li);
        const int d = (int)kc->dims[4], Hkv = (int)kc->dims[2];
        SHAPE_CHECK(qn->dims[0] == d && kn->dims[0] == d, "layer %d: norm weights must have head_dim %d", li, d);
        SHAPE_CHECK(q->dims[1] % d == 0 && k->dims[1] == (int64_t)Hkv * d && v->dims[1] == k->dims[1],
                    "layer %d: q %s k %s v %s vs Hkv=%d d=%d", li, dims_str(q->dims).c_str(), dims_str(k->dims).c_str(),
                    dims_str(v->dims).c_str(), Hkv, d);
        const int Hq = (int)(q->dims[1] / d);
        SHAPE_CHECK(Hq % Hkv == 0, "layer %d: %d query heads not a multiple of %d kv heads", li, Hq, Hkv);
        SHAPE_CHECK(o->dims[1] == q->dims[1], "layer %d: o %s vs q %s", li, dims_str(o->dims).c_str(),
                    dims_str(q->dims).c_str());
        if (R < 0) R = (int)q->dims[0];
        // requests of the cache: its second extent, or the page table's rows
        const int64_t creq = PG ? kvp->dims[0] : kc->dims[1];
        if (Rq < 0) Rq = (int)creq;
        SHAPE_CHECK(q->dims[0] == R && k->dims[0] == R && v->dims[0] == R && o->dims[0] == R &&
                        creq == (PF ? Rq : R),
                    "layer %d: request count mismatch (graph %d, cache %lld)", li, R, (long long)creq);
        if (PG)
          SHAPE_CHECK(kc->dims[3] == PG, "layer %d: paged caches %s need pages of kv_page_size = %d positions", li,
                      dims_str(kc->dims).c_str(), PG);
        SHAPE_CHECK(Ly.layer >= 0 && Ly.layer < kc->dims[0], "layer %d: cache layer %d out of range %lld", li, Ly.layer,
                    (long long)kc->dims[0]);
        const int G = Hq / Hkv;
        const bool okGd = (d == 64 || d == 128) && (G == 1 || G == 2 || G == 4);
        if (!okGd)
          return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: head_dim %d with %d query heads per kv head", li, d, G);
        const int gx = Ly.grid_dim.x, gy = Ly.grid_dim.y > 0 ? Ly.grid_dim.y : 1, gz = Ly.grid_dim.z > 0 ? Ly.grid_dim.z : 1;
        SHAPE_CHECK(gx == Hkv && gz == R, "layer %d: ATTENTION needs grid_dim = (kv_heads=%d, chunks, requests=%d)", li,
                    Hkv, R);
        SHAPE_CHECK(gy >= 1 && gy <= MAX_SPLIT_CHUNKS, "layer %d: %d attention chunks (1..%d)", li, gy,
                    MAX_SPLIT_CHUNKS);
        op.Hq = Hq; op.Hkv = Hkv; op.d = d; op.G = G; op.C = gy;
        op.L = (int)kc->dims[0];
        op.S = PG ? (int)(kvp->dims[1] * PG) : (int)kc->dims[3];  // positions per request
        if (PG) {
          op.page = PG;
          op.npages = (int)kc->dims[1];
          op.max_pages = (int)kvp->dims[1];
          op.kv_pages = (const int32_t*)kvp->ptr;
        }
        op.layer = Ly.layer;
        op.q = (const uint64_t*)q->ptr; op.k = (const uint64_t*)k->ptr; op.v = (const uint64_t*)v->ptr;
        op.qn_w = (const uint16_t*)qn->ptr; op.kn_w = (const uint16_t*)kn->ptr;
        op.kc = (uint16_t*)kc->ptr; op.vc = (uint16_t*)vc->ptr;
        op.a_out = (uint64_t*)o->ptr;
        op.N = Hq * d;
        if (c->S_cache == 0 || op.S < c->S_cache) c->S_cache = op.S;
        part_floats = std::max(part_floats, (size_t)R * Hq * gy * (d + 2));
        merge_off[li] = {1, merge_u32};
        merge_u32 += (size_t)R * Hkv;
        const float theta = Ly.rope_theta > 0 ? Ly.rope_theta : 1.0e6f;
        int ri = -1;
        for (size_t i = 0; i < rope_keys.size(); ++i)
          if (rope_keys[i].theta == theta && rope_keys[i].d == d && rope_keys[i].S == op.S) ri = (int)i;
        if (ri < 0) { rope_keys.push_back({theta, d, op.S}); ri = (int)rope_keys.size() - 1; }
        rope_of[li] = ri;
        int rc = check_grid(c, li, Ly, ntasks, 0);
        if (rc != MPK_OK) return rc;
        op.signal_per_task = 0;
        op.out_trigger = R * Hkv;
        if (L < 0 || op.L > L) L = op.L;
        break;
      }
      case MPK_OP_RMSNORM_QKV_ATTENTION: {
        op.kind = TK_QKV_ATTN;
        if (PG)
          return fail(c, MPK_ERR_UNSUPPORTED,
                      "layer %d: the fused projections + attention operation needs a contiguous KV cache (kv_page_size "
                      "= 0); paged caches take RMSNORM_LINEAR + ATTENTION", li);
        const Tensor *x, *wn, *wq, *wk, *wv, *qn, *kn, *kc, *vc, *q, *k, *v, *o;
        NEED("inputs[0] (x)", Ly.inputs[0], MPK_FP32T, 2, &x);
        NEED("weights[0] (norm)", Ly.weights[0], MPK_BF16, 1, &wn);
        NEED("weights[1] (Wq)", Ly.weights[1], MPK_BF16, 2, &wq);
        NEED("weights[2] (Wk)", Ly.weights[2], MPK_BF16, 2, &wk);
        NEED("weights[3] (Wv)", Ly.weights[3], MPK_BF16, 2, &wv);
        NEED("weights[4] (q_norm)", Ly.weights[4], MPK_BF16, 1, &qn);
        NEED("weights[5] (k_norm)", Ly.weights[5], MPK_BF16, 1, &kn);
        NEED("weights[6] (k_cache)", Ly.weights[6], MPK_BF16, 5, &kc);
        NEED("weights[7] (v_cache)", Ly.weights[7], MPK_BF16, 5, &vc);
        NEED("outputs[0] (q)", Ly.outputs[0], MPK_FP32T, 2, &q);
        NEED("outputs[1] (k)", Ly.outputs[1], MPK_FP32T, 2, &k);
        NEED("outputs[2] (v)", Ly.outputs[2], MPK_FP32T, 2, &v);
        NEED("outputs[3] (o)", Ly.outputs[3], MPK_FP32T, 2, &o);
        op.K = (int)x->dims[1];
        SHAPE_CHECK(wn->dims[0] == op.K, "layer %d: norm weight %s, input width %d", li, dims_str(wn->dims).c_str(), op.K);
        SHAPE_CHECK(kc->dims == vc->dims, "layer %d: k/v caches differ", li);
        const int d = (int)kc->dims[4], Hkv = (int)kc->dims[2];
        SHAPE_CHECK(wq->dims[0] % d == 0, "layer %d: Wq rows %lld not a multiple of head_dim %d", li,
                    (long long)wq->dims[0], d);
        const int Hq = (int)(wq->dims[0] / d);
        SHAPE_CHECK(Hq % Hkv == 0, "layer %d: %d query heads not a multiple of %d kv heads", li, Hq, Hkv);
        SHAPE_CHECK(wq->dims[1] == op.K && wk->dims[1] == op.K && wv->dims[1] == op.K &&
                        wk->dims[0] == (int64_t)Hkv * d && wv->dims[0] == (int64_t)Hkv * d,
                    "layer %d: Wq %s Wk %s Wv %s vs K=%d, Hkv=%d, d=%d", li, dims_str(wq->dims).c_str(),
                    dims_str(wk->dims).c_str(), dims_str(wv->dims).c_str(), op.K, Hkv, d);
        SHAPE_CHECK(qn->dims[0] == d && kn->dims[0] == d, "layer %d: norm weights must have head_dim %d", li, d);
        if (R < 0) R = (int)x->dims[0];
        if (Rq < 0) Rq = (int)kc->dims[1];
        SHAPE_CHECK(x->dims[0] == R && q->dims[0] == R && k->dims[0] == R && v->dims[0] == R && o->dims[0] == R &&
                        kc->dims[1] == R,
                    "layer %d: request count mismatch (graph %d)", li, R);
        SHAPE_CHECK(q->dims[1] == (int64_t)Hq * d && k->dims[1] == (int64_t)Hkv * d && v->dims[1] == k->dims[1] &&
                        o->dims[1] == q->dims[1],
                    "layer %d: q %s k %s v %s o %s", li, dims_str(q->dims).c_str(), dims_str(k->dims).c_str(),
                    dims_str(v->dims).c_str(), dims_str(o->dims).c_str());
        SHAPE_CHECK(Ly.layer >= 0 && Ly.layer < kc->dims[0], "layer %d: cache layer %d out of range", li, Ly.layer);
        if (R != 1)
          return fail(c, MPK_ERR_UNSUPPORTED,
                      "layer %d: the fused projections + attention operation serves one request (got %d); several "
                      "requests take RMSNORM_LINEAR + ATTENTION", li, R);
        const int G = Hq / Hkv;
        if (!((d == 64 || d == 128) && (G == 1 || G == 2 || G == 4)))
          return fail(c, MPK_ERR_UNSUPPORTED, "layer %d: head_dim %d with %d query heads per kv head", li, d, G);
        const int gx = Ly.grid_dim.x, gy = Ly.grid_dim.y > 0 ? Ly.grid_dim.y : 1,
                  gz = Ly.grid_dim.z > 0 ? Ly.grid_dim.z : 1;
        SHAPE_CHECK(gy == Hkv && gz == R,
                    "layer %d: RMSNORM_QKV_ATTENTION needs grid_dim = (tasks per kv head, kv_heads=%d, requests=%d)",
                    li, Hkv, R);
        op.groups = Hkv;
        op.N = G * d + 2 * d;
        SHAPE_CHECK(gx <= op.N, "layer %d: %d tasks per kv head for %d rows", li, gx, op.N);
        op.nseg = 3;
        op.seg_row0[0] = 0;
        op.seg_row0[1] = G * d;
        op.seg_row0[2] = G * d + d;
        op.seg_row0[3] = G * d + 2 * d;
        op.grp_rows[0] = G * d;
        op.grp_rows[1] = d;
        op.grp_rows[2] = d;
        op.W[0] = (const uint16_t*)wq->ptr;
        op.W[1] = (const uint16_t*)wk->ptr;
        op.W[2] = (const uint16_t*)wv->ptr;
        op.y[0] = (uint64_t*)q->ptr;
        op.y[1] = (uint64_t*)k->ptr;
        op.y[2] = (uint64_t*)v->ptr;
        op.x = (const uint64_t*)x->ptr;
        op.norm_w = (const uint16_t*)wn->ptr;
        op.Hq = Hq; op.Hkv = Hkv; op.d = d; op.G = G;
        op.L = (int)kc->dims[0];
        op.S = (int)kc->dims[3];
        op.layer = Ly.layer;
        op.q = op.y[0]; op.k = op.y[1]; op.v = op.y[2];
        op.qn_w = (const uint16_t*)qn->ptr; op.kn_w = (const uint16_t*)kn->ptr;
        op.kc = (uint16_t*)kc->ptr; op.vc = (uint16_t*)vc->ptr;
        op.a_out = (uint64_t*)o->ptr;
        if (c->S_cache == 0 || op.S < c->S_cache) c->S_cache = op.S;
        merge_off[li] = {1, merge_u32};
        merge_u32 += (size_t)R * Hkv;
        // group mode needs every task of the operation on its own worker
        op.group_sync = ntasks <= c->num_workers ? 1 : 0;
        // attention chunks per kv head (run by the group's first tasks); chunk
        // partials [Hkv][C][G][d + 2], written in both modes
        op.C = std::min(gx, MAX_GCHUNK);
        gpart_words = std::max(gpart_words, (size_t)Hkv * op.C * G * (d + 2));
        const float theta = Ly.rope_theta > 0 ? Ly.rope_theta : 1.0e6f;
        int ri = -1;
        for (size_t i = 0; i < rope_keys.size(); ++i)
          if (rope_keys[i].theta == theta && rope_keys[i].d == d && rope_keys[i].S == op.S) ri = (int)i;
        if (ri < 0) { rope_keys.push_back({theta, d, op.S}); ri = (int)rope_keys.size() - 1; }
        rope_of[li] = ri;
        int rc = gemv_geometry(c, li, op, false, true);
        if (rc != MPK_OK) return rc;
        rc = check_grid(c, li, Ly, ntasks, 0);
        if (rc != MPK_OK) return rc;
        op.signal_per_task = 0;
        op.out_trigger = R * Hkv;
        if (L < 0 || op.L > L) L = op.L;
        break;
      }
      default:
        return fail(c, MPK_ERR_INVALID_ARG, "layer %d: unknown op %d", li, Ly.op);
    }
  }
  if (R > MAX_REQUESTS)
    return fail(c, MPK_ERR_UNSUPPORTED, "%d requests (at most %d)", R, MAX_REQUESTS);
  if (n_argmax != 1 || ops[n_layers - 1].kind != TK_NORM_GEMV_ARGMAX)
    return fail(c, MPK_ERR_INVALID_ARG, "the graph must end with one RMSNORM_LMHEAD_ARGMAX operation");
  if (ops[0].kind != TK_EMBED)
    return fail(c, MPK_ERR_INVALID_ARG, "the graph must start with an EMBED operation");
  if (H < 0) H = ops[0].N;

  // events: op p signals event p; op p waits on event p-1 (op 0 on the last op,
  // one iteration behind).
  const int P = n_layers;

  // versions: for every tagged input, the operation that last wrote it earlier
  // in the iteration (a reader waits for that writer's tag)
  {
    std::map<const void*, int> writer;
    auto wr = [&](const void* b) {
      auto it = writer.find(b);
      return it == writer.end() ? -1 : it->second;
    };
    for (int p = 0; p < P; ++p) {
      OpDesc& op = ops[p];
      op.self = p;
      op.x_writer = -1;
      op.a_writer = -1;
      op.tagged = op.kind == TK_EMBED ? 0 : 1;
      switch (op.kind) {
        case TK_NORM_GEMV:
        case TK_NORM_GEMV_SILU:
        case TK_NORM_GEMV_ARGMAX:
        case TK_QKV_ATTN:
          op.x_writer = wr(op.x);
          if (op.kind == TK_QKV_ATTN) op.a_writer = p;
          break;
        case TK_GEMV_RESID:
          op.x_writer = wr(op.x_out);
          op.a_writer = wr(op.a_in);
          if (op.a_writer < 0)
            return fail(c, MPK_ERR_INVALID_ARG, "layer %d: its input is not written by an earlier operation", p);
          break;
        case TK_ATTN:
          op.a_writer = wr(op.q);
          if (op.a_writer < 0 || wr(op.k) != op.a_writer || wr(op.v) != op.a_writer)
            return fail(c, MPK_ERR_INVALID_ARG, "layer %d: q, k and v must come from one earlier operation", p);
          break;
        default:
          break;
      }
      if (op.kind != TK_EMBED && op.kind != TK_ATTN && op.x_writer < 0)
        return fail(c, MPK_ERR_INVALID_ARG, "layer %d: its x is not written by an earlier operation", p);
      switch (op.kind) {
        case TK_EMBED:
        case TK_GEMV_RESID:
          writer[op.x_out] = p;
          break;
        case TK_NORM_GEMV:
          for (int sg = 0; sg < op.nseg; ++sg) writer[op.y[sg]] = p;
          break;
        case TK_QKV_ATTN:
          for (int sg = 0; sg < 3; ++sg) writer[op.y[sg]] = p;
          writer[op.a_out] = p;
          break;
        case TK_NORM_GEMV_SILU:
        case TK_ATTN:
          writer[op.a_out] = p;
          break;
        default:
          break;
      }
    }
  }
  // Projections may be claimed dynamically: an op's tasks are shared out by a
  // counter, so workers that finish the previous op early take them first and
  // a worker that runs late takes fewer (or, with fewer tasks than workers,
  // none).  The tensor-core projections over several requests always are (a
  // late worker would otherwise stay late: the last segment task of a split
  // reduction to arrive runs the row block's epilogue); the one-request GEMV
  // operations when the options ask for it.  Attention keeps its fixed
  // task-to-worker mapping (the fused op's group tasks wait on one another).
  for (int p = 0; p < P; ++p) {
    OpDesc& op = ops[p];
    const bool proj = op.kind == TK_NORM_GEMV || op.kind == TK_GEMV_RESID || op.kind == TK_NORM_GEMV_SILU ||
                      op.kind == TK_NORM_GEMV_ARGMAX;
    op.dynamic = proj && (op.batched || o.dynamic_tasks > 0) ? 1 : 0;
    if (op.dynamic && op.ntasks >= (int)TASK_CLAIM)
      return fail(c, MPK_ERR_INVALID_ARG, "layer %d: at most %u tasks", p, TASK_CLAIM - 1);
  }
  c->zero_each_run.clear();
  for (auto& kv : c->tensors)
    if (kv.second.dtype == MPK_FP32T) {
      size_t n = 1;
      for (int64_t d : kv.second.dims) n *= (size_t)d;
      c->zero_each_run.push_back({kv.second.ptr, n * 8});
    }
  for (int p = 0; p < P; ++p) {
    ops[p].out_event = p;
    const int dp = (p + P - 1) % P;
    ops[p].dep_event = dp;
    ops[p].dep_trigger = ops[dp].out_trigger;
    ops[p].dep_iter_offset = p == 0 ? 0 : 1;
  }
  if (o.debug_stall_op > 0) {
    const int p = o.debug_stall_op - 1;
    if (p >= P)
      return fail(c, MPK_ERR_INVALID_ARG, "debug_stall_op %d beyond the %d operations", o.debug_stall_op, P);
    if (ops[p].tagged) {
      // wait for the versions of the next iteration, which only this op's own
      // completion could lead to
      ops[p].tag_skew = (uint32_t)P;
    } else {
      // one more completion per iteration than the dependency ever delivers
      ops[p].dep_trigger += 1;
      ops[p].dep_iter_offset = 1;
    }
  }

  // ---- workspace
  // sync block (zeroed before every run): events | q_head | q_tail | ctl | status | keys | arrive | merge counters |
  // timeline_n | split row-block counters
  const size_t line = EVENT_STRIDE * sizeof(uint32_t);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o2 = off; off += (bytes + 127) / 128 * 128; return o2; };
  const size_t o_events = take(line * P);
  const size_t o_claims = take(line * P * CLAIM_SLOTS);
  const size_t o_qhead = take(line * c->num_workers);
  const size_t o_qtail = take(line * c->num_workers);
  const size_t o_ctl = take(sizeof(Control));
  const size_t o_status = take(sizeof(Status));
  const size_t o_keys = take(sizeof(unsigned long long) * (size_t)R);
  const size_t o_arrive = take(line);
  const size_t o_merge = take(sizeof(uint32_t) * (merge_u32 ? merge_u32 : 1));
  const size_t o_tln = take(line);
  const size_t o_blk = take(sizeof(uint32_t) * (blk_u32 ? blk_u32 : 1));
  // batched projections with a split reduction: their own row-block counters
  // and partial sums per operation (consecutive projections can overlap)
  std::vector<size_t> bblk_off(P, 0), bpart_off(P, 0);
  size_t bblk_u32 = 0, bpart_floats = 0;
  for (int p = 0; p < P; ++p) {
    const OpDesc& op = ops[p];
    if (!op.batched || op.bsplit <= 1) continue;
    bblk_off[p] = bblk_u32;
    bblk_u32 += (size_t)op.nb;
    bpart_off[p] = bpart_floats;
    bpart_floats += (size_t)op.bsplit * op.N * batch_width(R) * (op.kind == TK_NORM_GEMV_SILU ? 2 : 1);
  }
  const size_t o_bblk = take(sizeof(uint32_t) * (bblk_u32 ? bblk_u32 : 1));
  c->sync_bytes = off;
  uint8_t* sb = nullptr;
  int rc = alloc(c, &sb, off);
  if (rc != MPK_OK) return rc;
  c->sync_block = sb;
  unsigned long long* queue = nullptr;
  rc = alloc(c, &queue, sizeof(unsigned long long) * QUEUE_CAP * c->num_workers);
  if (rc != MPK_OK) return rc;
  float* part = nullptr;
  rc = alloc(c, &part, sizeof(float) * (part_floats ? part_floats : 1));
  if (rc != MPK_OK) return rc;
  uint64_t* kpart = nullptr;
  rc = alloc(c, &kpart, sizeof(uint64_t) * (kpart_floats ? kpart_floats : 1));
  if (rc != MPK_OK) return rc;
  c->zero_each_run.push_back({kpart, sizeof(uint64_t) * (kpart_floats ? kpart_floats : 1)});
  uint64_t* gpart = nullptr;
  rc = alloc(c, &gpart, sizeof(uint64_t) * (gpart_words ? gpart_words : 1));
  if (rc != MPK_OK) return rc;
  c->zero_each_run.push_back({gpart, sizeof(uint64_t) * (gpart_words ? gpart_words : 1)});
  std::vector<float2*> rope_dev(rope_keys.size(), nullptr);
  for (size_t i = 0; i < rope_keys.size(); ++i) {
    const RopeKey& k = rope_keys[i];
    std::vector<float2> tab((size_t)k.S * (k.d / 2));
    for (int s = 0; s < k.S; ++s)
      for (int j = 0; j < k.d / 2; ++j) {
        const double ang = (double)s * std::pow((double)k.theta, -2.0 * j / (double)k.d);
        tab[(size_t)s * (k.d / 2) + j] = make_float2((float)std::cos(ang), (float)std::sin(ang));
      }
    rc = alloc(c, &rope_dev[i], tab.size() * sizeof(float2));
    if (rc != MPK_OK) return rc;
    CUDA_OR_FAIL(c, cudaMemcpy(rope_dev[i], tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice));
  }
  float* bpart = nullptr;
  if (bpart_floats) {
    rc = alloc(c, &bpart, sizeof(float) * bpart_floats);
    if (rc != MPK_OK) return rc;
  }
  // tensor maps of the batched projections' weights and of the caches the
  // split-K attention streams (64-byte aligned device copies)
  std::vector<CUtensorMap> tmaps;
  std::vector<std::pair<int, int>> tmap_of;  // (op, slot): slot MAX_SEG = the up matrix, -1 / -2: k / v cache
  for (int p = 0; p < P; ++p) {
    const OpDesc& op = ops[p];
    if (op.kind == TK_ATTN) {
      const int64_t rows = op.page > 0 ? (int64_t)op.L * op.npages * op.Hkv * op.page
                                       : (int64_t)op.L * Rq * op.Hkv * op.S;
      if (rows >= ((int64_t)1 << 31))
        return fail(c, MPK_ERR_UNSUPPORTED, "op %d: a KV cache of %lld rows of d (at most 2^31 - 1)", p,
                    (long long)rows);
      for (int w = 0; w < 2; ++w) {
        CUtensorMap m;
        rc = make_weight_map(c, p, &m, w == 0 ? op.kc : op.vc, rows, op.d, STAGE_BYTES / (4 * op.d));
        if (rc != MPK_OK) return rc;
        tmaps.push_back(m);
        tmap_of.push_back({p, -1 - w});
      }
      continue;
    }
    if (!op.batched) continue;
    for (int sg = 0; sg <= MAX_SEG; ++sg) {
      const void* w = sg < MAX_SEG ? (sg < op.nseg ? op.W[sg] : nullptr)
                                   : (op.kind == TK_NORM_GEMV_SILU ? op.W_up : nullptr);
      if (!w) continue;
      const int64_t rows = (sg < MAX_SEG && op.nseg > 1) ? op.grp_rows[sg] : op.N;
      CUtensorMap m;
      rc = make_weight_map(c, p, &m, w, rows, op.K);
      if (rc != MPK_OK) return rc;
      tmaps.push_back(m);
      tmap_of.push_back({p, sg});
    }
  }
  if (!tmaps.empty()) {
    CUtensorMap* tm_dev = nullptr;
    rc = alloc(c, &tm_dev, sizeof(CUtensorMap) * tmaps.size());
    if (rc != MPK_OK) return rc;
    CUDA_OR_FAIL(c, cudaMemcpy(tm_dev, tmaps.data(), sizeof(CUtensorMap) * tmaps.size(), cudaMemcpyHostToDevice));
    for (size_t i = 0; i < tmap_of.size(); ++i) {
      OpDesc& op = ops[tmap_of[i].first];
      const int slot = tmap_of[i].second;
      if (slot == -1) op.tmap_kc = tm_dev + i;
      else if (slot == -2) op.tmap_vc = tm_dev + i;
      else if (slot < MAX_SEG) op.tmap[slot] = tm_dev + i;
      else op.tmap_up = tm_dev + i;
    }
  }
  for (int p = 0; p < P; ++p) {
    OpDesc& op = ops[p];
    if (op.batched && op.bsplit > 1) {
      op.bpart = bpart + bpart_off[p];
      op.blk_cnt = reinterpret_cast<uint32_t*>(sb + o_bblk) + bblk_off[p];
    }
  }
  if (R >= 2) {
    // per-block sums of squares of every residual stream (tagged, versioned
    // like the stream itself): one buffer per x tensor, published by its
    // writers, read by the RMSNorm operations
    std::map<const void*, uint64_t*> xss;
    for (int p = 0; p < P; ++p) {
      OpDesc& op = ops[p];
      if (op.kind != TK_EMBED && op.kind != TK_GEMV_RESID) continue;
      uint64_t*& buf = xss[op.x_out];
      const size_t words = (size_t)((op.N + BM - 1) / BM) * R;
      if (!buf) {
        rc = alloc(c, &buf, words * sizeof(uint64_t));
        if (rc != MPK_OK) return rc;
        c->zero_each_run.push_back({buf, words * sizeof(uint64_t)});
      }
      op.xss_out = buf;
      op.xss_blocks = (op.N + BM - 1) / BM;
    }
    for (int p = 0; p < P; ++p) {
      OpDesc& op = ops[p];
      if (op.kind != TK_NORM_GEMV && op.kind != TK_NORM_GEMV_SILU && op.kind != TK_NORM_GEMV_ARGMAX) continue;
      auto it = xss.find(op.x);
      if (it == xss.end())
        return fail(c, MPK_ERR_INVALID_ARG, "layer %d: its input is written by no embedding or residual operation", p);
      op.xss_in = it->second;
      op.xss_blocks = (op.K + BM - 1) / BM;
    }
    // published input rows: every writer of x also writes, for the next
    // RMSNorm operation that reads this version of x, its rows as the
    // tensor-core input (bf16 hi/lo of x * that operation's norm weight, in
    // the swizzled shared-memory layout); one buffer per x tensor, zero in
    // the unused request rows and past the end of x
    std::map<const void*, uint16_t*> xb;
    for (int p = 0; p < P && o.poll_inputs <= 0; ++p) {
      OpDesc& op = ops[p];
      if (op.kind != TK_EMBED && op.kind != TK_GEMV_RESID) continue;
      int q = -1;
      for (int t = p + 1; t < P && q < 0; ++t) {
        if ((ops[t].kind == TK_EMBED || ops[t].kind == TK_GEMV_RESID) && ops[t].x_out == op.x_out) break;
        const bool norm = ops[t].kind == TK_NORM_GEMV || ops[t].kind == TK_NORM_GEMV_SILU ||
                          ops[t].kind == TK_NORM_GEMV_ARGMAX;
        if (norm && ops[t].x == op.x_out && ops[t].x_writer == p && ops[t].xb_in == nullptr) q = t;
      }
      if (q < 0) continue;
      uint16_t*& buf = xb[op.x_out];
      if (!buf) {
        const size_t bytes = (size_t)((op.N + BK - 1) / BK) * b_kblock_bytes(batch_width(R));
        rc = alloc(c, &buf, bytes);
        if (rc != MPK_OK) return rc;
      }
      op.xb_out = buf;
      op.xb_w = ops[q].norm_w;
      ops[q].xb_in = buf;
    }
    // published plain inputs of the o and down projections: the attention's
    // merge (flag per request and kv head) and the gate/up epilogue (flag per
    // row block) publish the rows; flags are tagged, so zeroed every run
    std::map<std::pair<const void*, int>, std::pair<uint16_t*, uint64_t*>> ab;
    for (int q = 0; q < P && o.poll_inputs <= 0; ++q) {
      OpDesc& rd = ops[q];
      if (rd.kind != TK_GEMV_RESID || !rd.batched || rd.a_writer < 0) continue;
      OpDesc& wr = ops[rd.a_writer];
      int grp, rstride;
      size_t nflags;
      if (wr.kind == TK_ATTN) {
        grp = wr.G * wr.d;
        rstride = wr.Hkv;
        nflags = (size_t)R * wr.Hkv;
      } else if (wr.kind == TK_NORM_GEMV_SILU && wr.batched) {
        grp = BM;
        rstride = 0;
        nflags = (size_t)((wr.N + BM - 1) / BM);
      } else {
        continue;
      }
      if (wr.xb_out != nullptr || rd.K % BK != 0 || grp % BK != 0) continue;
      auto& e = ab[{rd.a_in, wr.kind}];
      if (!e.first) {
        rc = alloc(c, &e.first, (size_t)(rd.K / BK) * b_kblock_bytes(batch_width(R)));
        if (rc != MPK_OK) return rc;
        rc = alloc(c, &e.second, nflags * sizeof(uint64_t));
        if (rc != MPK_OK) return rc;
        c->zero_each_run.push_back({e.second, nflags * sizeof(uint64_t)});
      }
      wr.xb_out = e.first;
      wr.xb_w = nullptr;
      wr.xf_out = e.second;
      rd.xb_in = e.first;
      rd.xf_in = e.second;
      rd.xf_grp = grp;
      rd.xf_rstride = rstride;
    }
  }
  unsigned long long* timeline = nullptr;
  if (o.profiling) {
    rc = alloc(c, &timeline, sizeof(unsigned long long) * TIMELINE_FIELDS * (size_t)o.max_timeline);
    if (rc != MPK_OK) return rc;
  }
  for (int p = 0; p < P; ++p) {
    OpDesc& op = ops[p];
    if (op.kind == TK_ATTN) {
      op.part = part;
      op.merge_cnt = reinterpret_cast<uint32_t*>(sb + o_merge) + merge_off[p].second;
      op.rope = rope_dev[rope_of[p]];
    }
    if (op.kind == TK_QKV_ATTN) {
      op.gpart = gpart;  // one group-mode operation at a time uses it
      op.grp_cnt = reinterpret_cast<uint32_t*>(sb + o_merge) + merge_off[p].second;
      op.rope = rope_dev[rope_of[p]];
    }
    if (op.ksplit > 1) {
      // shared by every split projection: they run one after another
      op.kpart = kpart;
      op.blk_cnt = reinterpret_cast<uint32_t*>(sb + o_blk);
    }
    if (op.kind == TK_NORM_GEMV_ARGMAX) {
      op.keys = reinterpret_cast<unsigned long long*>(sb + o_keys);
      op.arrive = reinterpret_cast<uint32_t*>(sb + o_arrive);
    }
  }
  rc = alloc(c, &c->ops_dev, sizeof(OpDesc) * P);
  if (rc != MPK_OK) return rc;
  CUDA_OR_FAIL(c, cudaMemcpy(c->ops_dev, ops.data(), sizeof(OpDesc) * P, cudaMemcpyHostToDevice));

  if (PF && (R != PF || R < 2 || R > MAX_PREFILL))
    return fail(c, MPK_ERR_SHAPE, "prefill_tokens = %d needs activations of that many rows (2..%d); the graph has %d",
                PF, MAX_PREFILL, R);
  if (!PF || Rq < 1) Rq = R;
  if (Rq > MAX_REQUESTS)
    return fail(c, MPK_ERR_UNSUPPORTED, "%d cached requests (at most %d)", Rq, MAX_REQUESTS);
  if (pred_rows >= 0 && pred_rows != Rq)
    return fail(c, MPK_ERR_SHAPE, "pred has %d rows, the graph serves %d requests", pred_rows, Rq);
  Graph& g = c->graph;
  memset(&g, 0, sizeof(g));
  g.ops = c->ops_dev;
  g.nops = P;
  g.batched = R >= 2 ? 1 : 0;
  g.bw = batch_width(R);
  g.split_attn = 0;
  for (int p = 0; p < P; ++p)
    if (ops[p].kind == TK_ATTN) g.split_attn = 1;
  g.R = R;
  g.V = V;
  g.H = H;
  g.L = L < 0 ? 0 : L;
  g.num_workers = c->num_workers;
  g.num_sched = c->num_local;
  g.sched_ctas = c->num_local / 4;
  g.lookahead = o.sched_lookahead;
  g.prefetch_bytes = o.prefetch_kb > 0 ? (uint32_t)o.prefetch_kb * 1024u : 0u;
  g.events = reinterpret_cast<uint32_t*>(sb + o_events);
  g.claims = reinterpret_cast<uint32_t*>(sb + o_claims);
  g.queue = queue;
  g.q_head = reinterpret_cast<uint32_t*>(sb + o_qhead);
  g.q_tail = reinterpret_cast<uint32_t*>(sb + o_qtail);
  g.ctl = reinterpret_cast<Control*>(sb + o_ctl);
  g.status = reinterpret_cast<Status*>(sb + o_status);
  uint32_t* abort_dev = nullptr;
  CUDA_OR_FAIL(c, cudaHostGetDevicePointer(reinterpret_cast<void**>(&abort_dev), c->abort_host, 0));
  g.abort_flag = reinterpret_cast<volatile int32_t*>(abort_dev);
  g.timeout_ns = (uint64_t)(o.timeout_s * 1e9);
  g.profiling = o.profiling;
  g.max_timeline = o.max_timeline;
  g.timeline = timeline;
  g.timeline_n = reinterpret_cast<uint32_t*>(sb + o_tln);
  c->status_dev = g.status;
  c->R = R;
  c->V = V;
  c->H = H;
  c->L = g.L;
  c->pred_S = S;
  c->prefill = PF;
  c->Rq = Rq;
  g.prefill = PF ? 1 : 0;
  g.Rq = Rq;
  c->ops = ops;
  c->compiled = true;
  return MPK_OK;
}

static int prepare_run(mpk_ctx* c, int32_t* step, int64_t* tokens, const int32_t* step_end, int64_t seq_len,
                       cudaStream_t s) {
  if (!c) return MPK_ERR_INVALID_ARG;
  if (!c->compiled) return fail(c, MPK_ERR_STATE, "mpk_run before mpk_compile");
  if (!step || !tokens) return fail(c, MPK_ERR_INVALID_ARG, "step and tokens are required");
  if (seq_len < 2) return fail(c, MPK_ERR_INVALID_ARG, "seq_length %lld < 2", (long long)seq_len);
  if (c->S_cache > 0 && seq_len - 1 > c->S_cache)
    return fail(c, MPK_ERR_SHAPE, "seq_length %lld needs %lld cached positions, the KV cache holds %d",
                (long long)seq_len, (long long)seq_len - 1, c->S_cache);
  if (c->pred_S > 0 && c->pred_S != seq_len)
    return fail(c, MPK_ERR_SHAPE, "pred has %d columns, tokens %lld", c->pred_S, (long long)seq_len);
  Graph& g = c->graph;
  g.step = step;
  g.tokens = tokens;
  g.step_end = step_end;
  g.S = (int32_t)seq_len;
  g.capture_iter = c->capture_iter;
  g.cap_logits = c->cap_logits;
  g.cap_hidden = c->cap_hidden;
  CUDA_OR_FAIL(c, cudaMemsetAsync(c->sync_block, 0, c->sync_bytes, s));
  for (const auto& z : c->zero_each_run) CUDA_OR_FAIL(c, cudaMemsetAsync(z.first, 0, z.second, s));
  return MPK_OK;
}

int mpk_run(mpk_ctx* c, int32_t* step, int64_t* tokens, int num_requests, int64_t seq_len,
            const int32_t* step_end, void* stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (c && c->compiled && num_requests != c->Rq)
    return fail(c, MPK_ERR_SHAPE, "tokens has %d requests, the graph %d", num_requests, c->Rq);
  int rc = prepare_run(c, step, tokens, step_end, seq_len, s);
  if (rc != MPK_OK) return rc;
  *(volatile int32_t*)c->abort_host = 0;
  c->graph.op_by_op = 0;
  CUDA_OR_FAIL(c, launch_persistent(c->graph, c->sms, s));
  return MPK_OK;
}

int mpk_run_op_by_op(mpk_ctx* c, int32_t* step, int64_t* tokens, int num_requests, int64_t seq_len,
                     const int32_t* step_end, void* stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int nreq = c && c->compiled ? c->Rq : 0;
  if (c && c->compiled && num_requests != nreq)
    return fail(c, MPK_ERR_SHAPE, "tokens has %d requests, the graph %d", num_requests, nreq);
  int rc = prepare_run(c, step, tokens, step_end, seq_len, s);
  if (rc != MPK_OK) return rc;
  // The host needs the iteration count: read step / step_end.
  std::vector<int32_t> st(nreq), se(nreq, (int32_t)(seq_len - 1));
  CUDA_OR_FAIL(c, cudaMemcpyAsync(st.data(), step, sizeof(int32_t) * nreq, cudaMemcpyDeviceToHost, s));
  if (step_end)
    CUDA_OR_FAIL(c, cudaMemcpyAsync(se.data(), step_end, sizeof(int32_t) * nreq, cudaMemcpyDeviceToHost, s));
  CUDA_OR_FAIL(c, cudaStreamSynchronize(s));
  int64_t n_iter = 0;
  for (int r = 0; r < nreq; ++r) {
    const int64_t end = std::min<int64_t>(se[r], seq_len - 1);
    if (st[r] >= 0 && st[r] < end) {
      const int64_t left = end - st[r];
      // prefill: the requests one after another, R positions per iteration
      n_iter = c->prefill ? n_iter + (left + c->R - 1) / c->R : std::max<int64_t>(n_iter, left);
    }
  }
  c->graph.op_by_op = 1;
  for (int64_t it = 0; it < n_iter; ++it)
    for (int p = 0; p < (int)c->ops.size(); ++p)
      CUDA_OR_FAIL(c, launch_op(c->graph, p, c->ops[p].ntasks, (uint32_t)it, c->ops[p].group_sync != 0, s));
  c->graph.op_by_op = 0;
  return MPK_OK;
}

int mpk_set_capture(mpk_ctx* c, int iter, float* logits, float* hidden) {
  if (!c) return MPK_ERR_INVALID_ARG;
  c->capture_iter = iter;
  c->cap_logits = logits;
  c->cap_hidden = hidden;
  return MPK_OK;
}

int mpk_status(mpk_ctx* c) {
  if (!c) return MPK_ERR_INVALID_ARG;
  if (!c->compiled) return MPK_OK;
  Status st{};
  cudaError_t e = cudaMemcpy(&st, c->status_dev, sizeof(st), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(c, MPK_ERR_CUDA, "status read failed: %s", cudaGetErrorString(e));
  if (st.code == 0) return MPK_OK;
  static const char* where[] = {"?", "worker dependency wait", "producer queue wait", "weight ring wait",
                                "task fifo wait", "scheduler gate wait", "scheduler queue space wait", "start",
                                "embedding token check", "task dispatch", "iteration boundary",
                                "tagged input wait", "KV page table check"};
  const char* w = (st.where >= 0 && st.where < 13) ? where[st.where] : "?";
  fail(c, st.code, "device status %d at %s: op %d task %d worker %d iter %d observed %u expected %u", st.code, w, st.op,
       st.task, st.worker, st.iter, st.observed, st.expected);
  return st.code;
}

int mpk_request_abort(mpk_ctx* c) {
  if (!c || !c->abort_host) return MPK_ERR_INVALID_ARG;
  *(volatile int32_t*)c->abort_host = 1;
  return MPK_OK;
}

int mpk_timeline(mpk_ctx* c, uint64_t* out, int cap) {
  if (!c) return MPK_ERR_INVALID_ARG;
  if (!c->compiled || !c->graph.timeline) return 0;
  uint32_t n = 0;
  CUDA_OR_FAIL(c, cudaMemcpy(&n, c->graph.timeline_n, sizeof(n), cudaMemcpyDeviceToHost));
  if ((int)n > c->graph.max_timeline) n = (uint32_t)c->graph.max_timeline;
  if (out && cap > 0) {
    const size_t k = std::min<size_t>(n, (size_t)cap);
    CUDA_OR_FAIL(c, cudaMemcpy(out, c->graph.timeline, k * TIMELINE_FIELDS * sizeof(uint64_t), cudaMemcpyDeviceToHost));
  }
  return (int)n;
}

int mpk_destroy(mpk_ctx* c) {
  if (!c) return MPK_ERR_INVALID_ARG;
  for (void* p : c->allocs) cudaFree(p);
  if (c->abort_host) cudaFreeHost(c->abort_host);
  delete c;
  return MPK_OK;
}

const char* mpk_last_error(mpk_ctx* c) { return c ? c->err.c_str() : g_create_error.c_str(); }

}  // extern "C"
