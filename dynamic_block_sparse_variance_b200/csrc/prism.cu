// C ABI of the Prism sparse-attention library (declared in include/prism.h).
// The whole library is this one translation unit: it includes the kernel
// headers, validates arguments on the host, lays out workspaces and launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <mutex>
#include <string>

#include "attn_mma_bwd.cuh"
#include "attn_tc_bwd.cuh"
#include "indicator.cuh"
#include "norms.cuh"
#include "permute.cuh"
#include "select.cuh"

namespace prism {

static thread_local std::string t_error;
static int g_attn_backend = 0;
static uint32_t g_wait_limit = 0;
static int g_debug_stall = 0;
constexpr uint32_t kDefaultWaitLimit = 1u << 22;

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over a [rows, 128] tensor of 16-bit elements (bf16 unless stated),
// 64 x 128 boxes, 128-byte swizzle; rows past the end read as zero.
static bool make_tile_map(CUtensorMap *map, const void *base, uint64_t rows,
                          CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128 * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
static prism_trace_fn g_trace = nullptr;
static void *g_trace_user = nullptr;

// Brackets one kernel launch with the trace hook (if any).
struct TraceScope {
  const char *name;
  cudaStream_t st;
  TraceScope(const char *n, cudaStream_t s) : name(n), st(s) {
    if (g_trace) g_trace(g_trace_user, name, 0, st);
  }
  ~TraceScope() {
    if (g_trace) g_trace(g_trace_user, name, 1, st);
  }
};
// Launches one kernel between the trace hooks and fails the call at once if
// the launch itself was rejected (a later successful call must not hide it).
#define PRISM_TRACED(NAME, ST, ...)                                                     \
  do {                                                                                  \
    cudaGetLastError();                                                                 \
    {                                                                                   \
      TraceScope _ts(NAME, ST);                                                         \
      __VA_ARGS__;                                                                      \
    }                                                                                   \
    const cudaError_t _le = cudaGetLastError();                                         \
    if (_le != cudaSuccess) return prism::fail(PRISM_ECUDA, cudaGetErrorString(_le));   \
  } while (0)

int fail(int code, const char *msg) {
  t_error = msg ? msg : "";
  return code;
}

struct Dims {
  int T, H, W, heads, D, ZT, ZY, ZX;
  int64_t N, Z, cap, C;
};

static int check_params(const prism_params *p, Dims *d) {
  if (!p) return fail(PRISM_EINVAL, "params is NULL");
  if (p->T <= 0 || p->H <= 0 || p->W <= 0 || p->T % kZone || p->H % kZone || p->W % kZone)
    return fail(PRISM_EINVAL, "token grid T, H, W must be positive multiples of 8");
  if (p->heads <= 0) return fail(PRISM_EINVAL, "heads must be positive");
  if (p->head_dim != 64 && p->head_dim != 128) return fail(PRISM_EINVAL, "head_dim must be 64 or 128");
  d->T = p->T; d->H = p->H; d->W = p->W; d->heads = p->heads; d->D = p->head_dim;
  d->ZT = p->T / kZone; d->ZY = p->H / kZone; d->ZX = p->W / kZone;
  d->N = (int64_t)p->T * p->H * p->W;
  d->Z = d->N / kZoneTokens;
  d->cap = d->Z * kMaxBlocksPerZone;
  d->C = (int64_t)p->heads * p->head_dim;
  if (d->Z > 65535) return fail(PRISM_EINVAL, "grid has more than 65535 macro-zones");
  if (p->fixed_shape < 0 || p->fixed_shape > 16) return fail(PRISM_EINVAL, "fixed_shape must be 0 or 1..16");
  if (!(p->sparsity >= 0.f && p->sparsity <= 1.f)) return fail(PRISM_EINVAL, "sparsity must be in [0, 1]");
  return PRISM_OK;
}

static bool aligned16(const void *ptr) { return ((uintptr_t)ptr & 15u) == 0; }
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
static cudaStream_t as_stream(prism_stream s) { return reinterpret_cast<cudaStream_t>(s); }
static float eff_scale(const prism_params *p) {
  return p->scale > 0.f ? p->scale : 1.f / std::sqrt((float)p->head_dim);
}

// Workspace layouts.
struct IndicatorWs {
  size_t part, rec, total;
  int nslab;
  IndicatorWs(const Dims &d) {
    nslab = (int)((d.C + kSlab - 1) / kSlab);
    part = 0;
    rec = align256((size_t)d.Z * nslab * 3 * sizeof(float));
    total = rec + align256((size_t)d.Z * kZoneRec * sizeof(double));
  }
};
struct SelectWs {
  size_t cnt, key, q, part, scores, fixed, per_head;
  int64_t R, nchunk;
  SelectWs(const Dims &d) {
    R = (int64_t)d.heads * d.cap;
    nchunk = (R + kScanChunk - 1) / kScanChunk;
    cnt = 0;
    key = cnt + align256(R * 4);
    q = key + align256(R * 4);
    part = q + align256(R * 4);
    scores = part + align256(nchunk * 8);
    fixed = scores;
    per_head = align256((size_t)d.cap * d.cap * sizeof(float));
  }
};
struct BwdWs {
  size_t delta, lse2, stat_inv, ccnt, col_ptr, fill, part, tot, row_idx, amax, f16, dqacc, total;
  int64_t R, nchunk;
  BwdWs(const Dims &d, int64_t col_capacity) {
    R = (int64_t)d.heads * d.cap;
    nchunk = (R + kScanChunk - 1) / kScanChunk;
    const size_t rows = (size_t)d.heads * d.N;
    // D, -LSE*log2e (warp-MMA path) or the integer shift m (tensor-core path),
    // and 2^(m - LSE*log2e): each padded by 128 entries for whole-tile bulk copies
    delta = 0;
    lse2 = align256((rows + 128) * 4);
    stat_inv = lse2 + align256((rows + 128) * 4);
    ccnt = stat_inv + align256((rows + 128) * 4);
    col_ptr = ccnt + align256(R * 4);
    fill = col_ptr + align256((R + 1) * 4);
    part = fill + align256(R * 4);
    tot = part + align256(nchunk * 8);
    row_idx = tot + 256;
    amax = row_idx + align256((size_t)(col_capacity > 0 ? col_capacity : 0) * 4);
    f16 = amax + align256((size_t)d.heads * 2 * 4);
    // head_dim 128 (tensor cores): fp16 copies of V and dO and the fp32 dQ accumulator
    dqacc = f16 + (d.D == 128 ? 2 * rows * 128 * 2 : 0);
    total = dqacc + (d.D == 128 ? rows * 128 * 4 : 0);
  }
};

// Forward (tensor-core path): per-head max |v| and V as scaled fp16.
struct FwdWs {
  size_t vmax, v16, total;
  explicit FwdWs(const Dims &d) {
    vmax = 0;
    v16 = align256((size_t)d.heads * 4);
    total = d.D == 128 ? v16 + (size_t)d.heads * d.N * 128 * 2 : 0;
  }
};

static int launch_scan(const int32_t *cnt, int64_t R, long long *part, int64_t nchunk, int64_t capacity,
                       int32_t *row_ptr, int64_t *nnz, cudaStream_t st) {
  PRISM_TRACED("scan_partial_kernel", st, scan_partial_kernel<<<(unsigned)nchunk, kScanThreads, 0, st>>>(cnt, R, part));
  PRISM_TRACED("scan_top_kernel", st, scan_top_kernel<<<1, kScanThreads, 0, st>>>(part, (int)nchunk, capacity, nnz));
  PRISM_TRACED("scan_final_kernel", st, scan_final_kernel<<<(unsigned)nchunk, kScanThreads, 0, st>>>(cnt, R, part, nnz, capacity, row_ptr));
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

}  // namespace prism

using namespace prism;

extern "C" {

const char *prism_last_error(void) { return t_error.c_str(); }

int prism_set_option(int option, int64_t value) {
  switch (option) {
    case PRISM_OPT_ATTN_BACKEND: g_attn_backend = (int)value; return PRISM_OK;
    case PRISM_OPT_WAIT_LIMIT: g_wait_limit = (uint32_t)value; return PRISM_OK;
    case PRISM_OPT_DEBUG_STALL: g_debug_stall = (int)value; return PRISM_OK;
    default: return fail(PRISM_EINVAL, "unknown option");
  }
}

int prism_set_trace(prism_trace_fn fn, void *user) {
  g_trace = fn;
  g_trace_user = user;
  return PRISM_OK;
}

int prism_device_status(prism_stream stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return fail(PRISM_ECUDA, cudaGetErrorString(e));
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int));
  if (e != cudaSuccess) return fail(PRISM_ECUDA, cudaGetErrorString(e));
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return fail(PRISM_ECUDA, cudaGetErrorString(e));
    const char *what = v == PRISM_ECAPACITY ? "selected pairs exceed col_capacity"
                       : v == PRISM_ETIMEOUT ? "a bounded device wait timed out"
                                             : "a device index check failed";
    return fail(v, what);
  }
  return PRISM_OK;
}

int prism_workspace_size(const prism_params *p, int kind, int64_t col_capacity, size_t *bytes,
                         size_t *bytes_all_heads) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if (!bytes) return fail(PRISM_EINVAL, "bytes is NULL");
  size_t all = 0;
  switch (kind) {
    case PRISM_WS_INDICATOR: *bytes = all = IndicatorWs(d).total; break;
    case PRISM_WS_SELECT: {
      SelectWs w(d);
      *bytes = w.fixed + w.per_head;
      all = w.fixed + w.per_head * d.heads;
      break;
    }
    case PRISM_WS_FWD: *bytes = all = FwdWs(d).total; break;
    case PRISM_WS_BWD: *bytes = all = BwdWs(d, col_capacity).total; break;
    default: return fail(PRISM_EINVAL, "unknown workspace kind");
  }
  if (bytes_all_heads) *bytes_all_heads = all;
  return PRISM_OK;
}

int prism_audio_norms(const void *h, int h_dtype, int64_t N, int C, float *a, prism_stream stream) {
  if (N < 0 || C <= 0) return fail(PRISM_EINVAL, "audio_norms: N must be >= 0 and C > 0");
  if (h_dtype != PRISM_BF16 && h_dtype != PRISM_F32) return fail(PRISM_EINVAL, "audio_norms: dtype must be bf16 or f32");
  if (C % (h_dtype == PRISM_BF16 ? 8 : 4)) return fail(PRISM_EINVAL, "audio_norms: C must fill whole 16-byte vectors");
  if (N == 0) return PRISM_OK;
  if (!h || !a) return fail(PRISM_EINVAL, "audio_norms: NULL argument");
  if (!aligned16(h)) return fail(PRISM_EINVAL, "audio_norms: h must be 16-byte aligned");
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows_per_block = kNormThreads / 32;
  const unsigned grid = (unsigned)std::min<int64_t>((N + rows_per_block - 1) / rows_per_block, (int64_t)sms * 8);
  cudaStream_t st = as_stream(stream);
  if (h_dtype == PRISM_BF16)
    PRISM_TRACED("audio_norms_kernel", st, audio_norms_kernel<__nv_bfloat16><<<grid, kNormThreads, 0, st>>>(
                                               static_cast<const __nv_bfloat16 *>(h), N, C, a));
  else
    PRISM_TRACED("audio_norms_kernel", st, audio_norms_kernel<float><<<grid, kNormThreads, 0, st>>>(
                                               static_cast<const float *>(h), N, C, a));
  return PRISM_OK;
}

int prism_zone_records(const prism_params *p, const void *V, int v_dtype, const float *audio, double *records,
                       void *workspace, size_t ws_bytes, prism_stream stream) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if (!V || !records) return fail(PRISM_EINVAL, "zone_records: V and records must be non-NULL");
  if (!aligned16(V)) return fail(PRISM_EINVAL, "V must be 16-byte aligned");
  if (v_dtype != PRISM_BF16 && v_dtype != PRISM_F32) return fail(PRISM_EINVAL, "V dtype must be bf16 or f32");
  IndicatorWs w(d);
  if (!workspace || ws_bytes < w.total) return fail(PRISM_EINVAL, "indicator workspace too small");
  cudaStream_t st = as_stream(stream);
  float *part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + w.part);
  dim3 grid(w.nslab, (unsigned)d.Z);
  if (v_dtype == PRISM_BF16)
    PRISM_TRACED("zone_stats_kernel", st, zone_stats_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(V), (int)d.C,
                                                            d.H, d.W, d.ZY, d.ZX, part));
  else
    PRISM_TRACED("zone_stats_kernel", st, zone_stats_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(V), (int)d.C, d.H, d.W, d.ZY,
                                                    d.ZX, part));
  PRISM_TRACED("zone_finish_kernel", st, zone_finish_kernel<<<(unsigned)d.Z, 64, 0, st>>>(part, w.nslab, (int)d.C, audio, d.H, d.W, d.ZY, d.ZX, records));
  return PRISM_OK;
}

int prism_zone_finalize(const prism_params *p, const double *records, int has_audio, float *g, float *rho,
                        float *debug, prism_stream stream) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if (!records || !g || !rho) return fail(PRISM_EINVAL, "zone_finalize: records, g and rho must be non-NULL");
  cudaStream_t st = as_stream(stream);
  PRISM_TRACED("zone_final_kernel", st, zone_final_kernel<<<1, 1024, 0, st>>>(records, (int)d.Z, has_audio != 0, p->eps, g, rho, debug));
  return PRISM_OK;
}

int prism_zone_indicator(const prism_params *p, const void *V, int v_dtype, const float *audio, float *g,
                         float *rho, float *debug, void *workspace, size_t ws_bytes, prism_stream stream) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if (!V || !g || !rho) return fail(PRISM_EINVAL, "V, g and rho must be non-NULL");
  if (!aligned16(V)) return fail(PRISM_EINVAL, "V must be 16-byte aligned");
  if (v_dtype != PRISM_BF16 && v_dtype != PRISM_F32) return fail(PRISM_EINVAL, "V dtype must be bf16 or f32");
  IndicatorWs w(d);
  if (!workspace || ws_bytes < w.total) return fail(PRISM_EINVAL, "indicator workspace too small");
  cudaStream_t st = as_stream(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *part = reinterpret_cast<float *>(ws + w.part);
  double *rec = reinterpret_cast<double *>(ws + w.rec);
  dim3 grid(w.nslab, (unsigned)d.Z);
  if (v_dtype == PRISM_BF16)
    PRISM_TRACED("zone_stats_kernel", st, zone_stats_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(V), (int)d.C,
                                                            d.H, d.W, d.ZY, d.ZX, part));
  else
    PRISM_TRACED("zone_stats_kernel", st, zone_stats_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(V), (int)d.C, d.H, d.W, d.ZY,
                                                    d.ZX, part));
  PRISM_TRACED("zone_finish_kernel", st, zone_finish_kernel<<<(unsigned)d.Z, 64, 0, st>>>(part, w.nslab, (int)d.C, audio, d.H, d.W, d.ZY, d.ZX, rec));
  PRISM_TRACED("zone_final_kernel", st, zone_final_kernel<<<1, 1024, 0, st>>>(rec, (int)d.Z, audio != nullptr, p->eps, g, rho, debug));
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

}  // extern "C"

// Scratch of prism_zone_indicator_noalloc: partial sums for up to
// PRISM_NOALLOC_MAX_ZONES zones x PRISM_NOALLOC_MAX_CHANNELS channels, laid
// out exactly like the indicator workspace.  Host code must not pass this
// name to a kernel (on the host it is only a stand-in); the device address is
// looked up once per device below.
constexpr size_t kNoallocPartBytes =
    (size_t)PRISM_NOALLOC_MAX_ZONES * (PRISM_NOALLOC_MAX_CHANNELS / kSlab) * 3 * sizeof(float);
constexpr size_t kNoallocBytes = kNoallocPartBytes + (size_t)PRISM_NOALLOC_MAX_ZONES * kZoneRec * sizeof(double);
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocBytes];

static std::mutex g_noalloc_mutex;
static void *g_noalloc_addr[256];   // per device ordinal

// Device address of the fixed scratch on the current device (looked up on the
// first call for that device and kept until exit; not valid across
// cudaDeviceReset, which the header states).
static int noalloc_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PRISM_ECUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= 256) return fail(PRISM_EINVAL, "device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return fail(PRISM_ECUDA, cudaGetErrorString(e));
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return PRISM_OK;
}

extern "C" {

int prism_zone_indicator_noalloc(const prism_params *p, const void *V, int v_dtype, const float *audio, float *g,
                                 float *rho, float *debug, prism_stream stream) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if (!V || !g || !rho) return fail(PRISM_EINVAL, "V, g and rho must be non-NULL");
  if (!aligned16(V)) return fail(PRISM_EINVAL, "V must be 16-byte aligned");
  if (v_dtype != PRISM_BF16 && v_dtype != PRISM_F32) return fail(PRISM_EINVAL, "V dtype must be bf16 or f32");
  if (d.Z > PRISM_NOALLOC_MAX_ZONES || d.C > PRISM_NOALLOC_MAX_CHANNELS)
    return fail(PRISM_EINVAL, "grid too large for the fixed scratch (see PRISM_NOALLOC_MAX_*)");
  IndicatorWs w(d);
  if (w.total > kNoallocBytes) return fail(PRISM_EINVAL, "grid too large for the fixed scratch");
  void *scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  uint8_t *ws = static_cast<uint8_t *>(scratch);
  // every partial and record is written before it is read, so nothing needs clearing
  float *part = reinterpret_cast<float *>(ws + w.part);
  double *rec = reinterpret_cast<double *>(ws + w.rec);
  dim3 grid(w.nslab, (unsigned)d.Z);
  if (v_dtype == PRISM_BF16)
    PRISM_TRACED("zone_stats_kernel", st, zone_stats_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(V), (int)d.C, d.H, d.W, d.ZY, d.ZX, part));
  else
    PRISM_TRACED("zone_stats_kernel", st, zone_stats_kernel<float><<<grid, 256, 0, st>>>(
        static_cast<const float *>(V), (int)d.C, d.H, d.W, d.ZY, d.ZX, part));
  PRISM_TRACED("zone_finish_kernel", st, zone_finish_kernel<<<(unsigned)d.Z, 64, 0, st>>>(
      part, w.nslab, (int)d.C, audio, d.H, d.W, d.ZY, d.ZX, rec));
  PRISM_TRACED("zone_final_kernel", st, zone_final_kernel<<<1, 1024, 0, st>>>(rec, (int)d.Z, audio != nullptr,
                                                                                p->eps, g, rho, debug));
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

int prism_assign_blocks(const prism_params *p, const float *g, const float *rho, uint8_t *shape_id,
                        int32_t *zone_blk_base, prism_block *blocks, int32_t *nblk, prism_stream stream) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if ((p->fixed_shape == PRISM_DYNAMIC_SHAPES && (!g || !rho)) || !shape_id || !zone_blk_base || !blocks || !nblk)
    return fail(PRISM_EINVAL, "assign_blocks: NULL argument");
  PRISM_TRACED("assign_blocks_kernel", as_stream(stream), assign_blocks_kernel<<<1, 1024, 0, as_stream(stream)>>>(g, rho, (int)d.Z, p->tau128, p->tau256, p->fixed_shape, shape_id,
                                                          zone_blk_base, blocks, nblk));
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

int prism_permute(const prism_params *p, const uint8_t *shape_id, const int32_t *zone_blk_base, const void *x,
                  int x_dtype, void *x_perm, float *pooled, prism_stream stream) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if (!shape_id || !x || !x_perm || (pooled && !zone_blk_base)) return fail(PRISM_EINVAL, "permute: NULL argument");
  if (!aligned16(x) || !aligned16(x_perm)) return fail(PRISM_EINVAL, "permute: tensors must be 16-byte aligned");
  if (x_dtype != PRISM_BF16 && x_dtype != PRISM_F32) return fail(PRISM_EINVAL, "permute: dtype must be bf16 or f32");
  cudaStream_t st = as_stream(stream);
  dim3 grid(d.heads, (unsigned)d.Z);
  auto *xp = static_cast<__nv_bfloat16 *>(x_perm);
#define PRISM_PERMUTE(TIN, DD)                                                                                \
  PRISM_TRACED("permute_kernel", st, permute_kernel<TIN, DD><<<grid, 256, 0, st>>>(static_cast<const TIN *>(x), d.heads, d.N, d.H, d.W, d.ZY, d.ZX, \
                                                shape_id, zone_blk_base, d.cap, xp, pooled))
  if (x_dtype == PRISM_BF16) {
    if (d.D == 128) PRISM_PERMUTE(__nv_bfloat16, 128); else PRISM_PERMUTE(__nv_bfloat16, 64);
  } else {
    if (d.D == 128) PRISM_PERMUTE(float, 128); else PRISM_PERMUTE(float, 64);
  }
#undef PRISM_PERMUTE
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

int prism_unpermute(const prism_params *p, const uint8_t *shape_id, const void *x_perm, int in_dtype, void *x,
                    int out_dtype, prism_stream stream) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if (!shape_id || !x || !x_perm) return fail(PRISM_EINVAL, "unpermute: NULL argument");
  if (!aligned16(x) || !aligned16(x_perm)) return fail(PRISM_EINVAL, "unpermute: tensors must be 16-byte aligned");
  if ((in_dtype != PRISM_BF16 && in_dtype != PRISM_F32) || (out_dtype != PRISM_BF16 && out_dtype != PRISM_F32))
    return fail(PRISM_EINVAL, "unpermute: dtype must be bf16 or f32");
  cudaStream_t st = as_stream(stream);
  dim3 grid(d.heads, (unsigned)d.Z);
#define PRISM_UNPERMUTE(TIN, TOUT, DD)                                                                        \
  PRISM_TRACED("unpermute_kernel", st, unpermute_kernel<TIN, TOUT, DD><<<grid, 256, 0, st>>>(static_cast<const TIN *>(x_perm), d.heads, d.N, d.H, \
                                                        d.W, d.ZY, d.ZX, shape_id, static_cast<TOUT *>(x)))
#define PRISM_UNPERMUTE_D(TIN, TOUT) \
  do { if (d.D == 128) PRISM_UNPERMUTE(TIN, TOUT, 128); else PRISM_UNPERMUTE(TIN, TOUT, 64); } while (0)
  if (in_dtype == PRISM_BF16 && out_dtype == PRISM_BF16) PRISM_UNPERMUTE_D(__nv_bfloat16, __nv_bfloat16);
  else if (in_dtype == PRISM_BF16) PRISM_UNPERMUTE_D(__nv_bfloat16, float);
  else if (out_dtype == PRISM_BF16) PRISM_UNPERMUTE_D(float, __nv_bfloat16);
  else PRISM_UNPERMUTE_D(float, float);
#undef PRISM_UNPERMUTE_D
#undef PRISM_UNPERMUTE
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

int prism_block_select(const prism_params *p, const int32_t *nblk, const float *q_pooled, const float *k_pooled,
                       int32_t *row_ptr, int32_t *col, int64_t col_capacity, int64_t *nnz, void *workspace,
                       size_t ws_bytes, prism_stream stream) {
  Dims d;
  int rc = check_params(p, &d);
  if (rc) return rc;
  if (!nblk || !q_pooled || !k_pooled || !row_ptr || !nnz || (!col && col_capacity > 0))
    return fail(PRISM_EINVAL, "block_select: NULL argument");
  if (!aligned16(q_pooled) || !aligned16(k_pooled)) return fail(PRISM_EINVAL, "block_select: pooled must be 16-byte aligned");
  if (p->sparsity == 0.f && p->top_k < 1) return fail(PRISM_EINVAL, "top_k must be >= 1");
  if (!(p->top_p > 0.f && p->top_p <= 1.f)) return fail(PRISM_EINVAL, "top_p must be in (0, 1]");
  const size_t key_bytes = (size_t)d.cap * 4;
  if (key_bytes + sizeof(SelShared) > 227 * 1024) return fail(PRISM_EINVAL, "too many blocks per head for selection");
  SelectWs w(d);
  if (!workspace || ws_bytes < w.fixed + w.per_head) return fail(PRISM_EINVAL, "select workspace too small");
  const int hp = (int)std::min<int64_t>(d.heads, (int64_t)((ws_bytes - w.fixed) / w.per_head));
  const bool once = hp >= d.heads;
  cudaStream_t st = as_stream(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *cnt = reinterpret_cast<int32_t *>(ws + w.cnt);
  uint32_t *ckey = reinterpret_cast<uint32_t *>(ws + w.key);
  int32_t *cq = reinterpret_cast<int32_t *>(ws + w.q);
  long long *part = reinterpret_cast<long long *>(ws + w.part);
  float *S = reinterpret_cast<float *>(ws + w.scores);
  const float scale = eff_scale(p);
  const unsigned tiles = (unsigned)((d.cap + 63) / 64);
  cudaFuncSetAttribute(row_cut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)key_bytes);
  for (int h0 = 0; h0 < d.heads; h0 += hp) {
    const int nh = std::min(hp, d.heads - h0);
    PRISM_TRACED("block_scores_kernel", st, block_scores_kernel<<<dim3(tiles, tiles, nh), 256, 0, st>>>(q_pooled, k_pooled, d.D, d.cap, nblk, h0, scale, S));
    PRISM_TRACED("row_cut_kernel", st, row_cut_kernel<<<dim3((unsigned)d.cap, nh), kSelThreads, key_bytes, st>>>(S, d.cap, nblk, h0, p->top_k,
                                                                               p->sparsity, p->top_p, cnt, ckey, cq));
  }
  PRISM_CUDA_CHECK_LAUNCH();
  rc = launch_scan(cnt, w.R, part, w.nchunk, col_capacity, row_ptr, nnz, st);
  if (rc) return rc;
  for (int h0 = 0; h0 < d.heads; h0 += hp) {
    const int nh = std::min(hp, d.heads - h0);
    if (!once)
      PRISM_TRACED("block_scores_kernel", st, block_scores_kernel<<<dim3(tiles, tiles, nh), 256, 0, st>>>(q_pooled, k_pooled, d.D, d.cap, nblk, h0, scale, S));
    PRISM_TRACED("emit_kernel", st, emit_kernel<<<dim3((unsigned)d.cap, nh), kSelThreads, 0, st>>>(S, d.cap, nblk, h0, ckey, cq, row_ptr, nnz,
                                                                  col_capacity, col));
  }
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

}  // extern "C"

static int check_attn(const prism_params *p, Dims *d, const void *blocks, const void *zbb, const void *nblk,
                      const void *const *tensors, int nt, const void *row_ptr, const void *col) {
  int rc = check_params(p, d);
  if (rc) return rc;
  if (!blocks || !zbb || !nblk || !row_ptr || !col) return fail(PRISM_EINVAL, "attention: NULL argument");
  for (int t = 0; t < nt; ++t) {
    if (!tensors[t]) return fail(PRISM_EINVAL, "attention: NULL tensor");
    if (!aligned16(tensors[t])) return fail(PRISM_EINVAL, "attention: tensors must be 16-byte aligned");
  }
  if (d->N / 64 > 0x7fffffffLL || d->heads > 65535) return fail(PRISM_EINVAL, "attention: grid too large");
  return PRISM_OK;
}

extern "C" {

int prism_bsa_fwd(const prism_params *p, const prism_block *blocks, const int32_t *zone_blk_base,
                  const int32_t *nblk, const void *q, const void *k, const void *v, const int32_t *row_ptr,
                  const int32_t *col, void *o, void *o_res, float *lse, void *workspace, size_t ws_bytes,
                  prism_stream stream) {
  Dims d;
  const void *tens[5] = {q, k, v, o, lse};
  int rc = check_attn(p, &d, blocks, zone_blk_base, nblk, tens, 5, row_ptr, col);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  const float scale_log2 = eff_scale(p) * kLog2e;
  dim3 grid((unsigned)(d.N / 64), d.heads);
  auto Q = static_cast<const __nv_bfloat16 *>(q), K = static_cast<const __nv_bfloat16 *>(k),
       Vv = static_cast<const __nv_bfloat16 *>(v);
  auto O = static_cast<__nv_bfloat16 *>(o);
  auto Ores = static_cast<__nv_bfloat16 *>(o_res);
  if (o_res && !aligned16(o_res)) return fail(PRISM_EINVAL, "attention: o_res must be 16-byte aligned");
  if (d.D == 128 && g_attn_backend == 0) {
    const FwdWs w(d);
    if (!workspace || ws_bytes < w.total || !aligned16(workspace))
      return fail(PRISM_EINVAL, "forward workspace missing, misaligned or below prism_workspace_size(PRISM_WS_FWD)");
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *vmax = reinterpret_cast<uint32_t *>(ws + w.vmax);
    void *v16 = ws + w.v16;
    // V -> fp16 scaled by 2^e_h per head (the PV product runs fp16 x fp16)
    const int64_t words = d.N * 16;   // 16-byte words per head
    const unsigned gx = (unsigned)std::max<int64_t>(1, std::min<int64_t>((words + 1023) / 1024, (148 * 8 + d.heads - 1) / d.heads));
    if (cudaMemsetAsync(vmax, 0, (size_t)d.heads * 4, st) != cudaSuccess)
      return fail(PRISM_ECUDA, "cudaMemsetAsync failed");
    PRISM_TRACED("head_absmax_kernel", st, head_absmax_kernel<<<dim3(gx, d.heads), 256, 0, st>>>(static_cast<const uint4 *>(v), words, vmax));
    PRISM_TRACED("v_to_f16_kernel", st, v_to_f16_kernel<<<dim3(gx, d.heads), 256, 0, st>>>(static_cast<const uint4 *>(v), words, vmax, static_cast<uint4 *>(v16)));
    CUtensorMap tq, tk, tv;
    const uint64_t rows = (uint64_t)d.heads * d.N;
    if (!make_tile_map(&tq, q, rows) || !make_tile_map(&tk, k, rows) ||
        !make_tile_map(&tv, v16, rows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
      return fail(PRISM_ECUDA, "cuTensorMapEncodeTiled failed");
    TcFwdArgs a;
    a.vmax = vmax;
    a.blocks = blocks;
    a.zone_blk_base = zone_blk_base;
    a.row_ptr = row_ptr;
    a.col = col;
    a.N = d.N;
    a.cap = d.cap;
    a.scale_log2 = scale_log2;
    a.o = O;
    a.o_res = Ores;
    a.lse = lse;
    a.wait_limit = g_wait_limit ? g_wait_limit : kDefaultWaitLimit;
    a.debug_stall = g_debug_stall;
    a.skip256 = g_debug_stall ? 0 : 1;   // the timeout test drives the single-tile kernel alone
    if (a.skip256) {
      cudaFuncSetAttribute(bsa_fwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTc2SmemBytes);
      dim3 pgrid((unsigned)(d.Z * 2), d.heads);
      PRISM_TRACED("bsa_fwd_tc2_kernel", st, bsa_fwd_tc2_kernel<<<pgrid, kTc2Threads, kTc2SmemBytes, st>>>(tq, tk, tv, a));
    }
    cudaFuncSetAttribute(bsa_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes);
    dim3 tgrid((unsigned)(d.Z * 8), d.heads);
    PRISM_TRACED("bsa_fwd_tc_kernel", st, bsa_fwd_tc_kernel<<<tgrid, 192, kTcSmemBytes, st>>>(tq, tk, tv, a));
  } else if (d.D == 128) {
    const int smem = 5 * 64 * 128 * 2;
    cudaFuncSetAttribute(bsa_fwd_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    PRISM_TRACED("bsa_fwd_mma_kernel", st, bsa_fwd_mma_kernel<128><<<grid, 128, smem, st>>>(Q, K, Vv, blocks, zone_blk_base, row_ptr, col, d.N, d.cap,
                                                     scale_log2, O, Ores, lse));
  } else {
    const int smem = 5 * 64 * 64 * 2;
    PRISM_TRACED("bsa_fwd_mma_kernel", st, bsa_fwd_mma_kernel<64><<<grid, 128, smem, st>>>(Q, K, Vv, blocks, zone_blk_base, row_ptr, col, d.N, d.cap,
                                                    scale_log2, O, Ores, lse));
  }
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

}  // extern "C"

template <int D>
static int launch_bwd_attn(const Dims &d, dim3 grid, cudaStream_t st, const __nv_bfloat16 *Q,
                            const __nv_bfloat16 *K, const __nv_bfloat16 *Vv, const __nv_bfloat16 *dO,
                            const float *lse, const float *delta, const prism_block *blocks,
                            const int32_t *zbb, const int32_t *row_ptr, const int32_t *col,
                            const int32_t *col_ptr, const int32_t *row_idx, float scale, __nv_bfloat16 *dq,
                            __nv_bfloat16 *dk, __nv_bfloat16 *dv) {
  const int smem_kv = 6 * 64 * D * 2 + 2 * 2 * 64 * 4;
  const int smem_q = 6 * 64 * D * 2;
  cudaFuncSetAttribute(bsa_dkdv_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv);
  cudaFuncSetAttribute(bsa_dq_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
  PRISM_TRACED("bsa_dkdv_mma_kernel", st, bsa_dkdv_mma_kernel<D><<<grid, 128, smem_kv, st>>>(Q, K, Vv, dO, lse, delta, blocks, zbb, col_ptr, row_idx,
                                                      d.N, d.cap, scale, dk, dv));
  PRISM_TRACED("bsa_dq_mma_kernel", st, bsa_dq_mma_kernel<D><<<grid, 128, smem_q, st>>>(Q, K, Vv, dO, lse, delta, blocks, zbb, row_ptr, col, d.N,
                                                   d.cap, scale, dq));
  return PRISM_OK;
}

extern "C" {

int prism_bsa_bwd(const prism_params *p, const prism_block *blocks, const int32_t *zone_blk_base,
                  const int32_t *nblk, const void *q, const void *k, const void *v, const void *o,
                  const void *o_res, const void *dout, const float *lse, const int32_t *row_ptr,
                  const int32_t *col,
                  const int64_t *nnz, int64_t col_capacity, void *dq, void *dk, void *dv, void *workspace,
                  size_t ws_bytes, prism_stream stream) {
  Dims d;
  const void *tens[10] = {q, k, v, o, dout, lse, dq, dk, dv, workspace};
  int rc = check_attn(p, &d, blocks, zone_blk_base, nblk, tens, 10, row_ptr, col);
  if (rc) return rc;
  if (!nnz) return fail(PRISM_EINVAL, "bwd: nnz is NULL");
  BwdWs w(d, col_capacity);
  if (ws_bytes < w.total) return fail(PRISM_EINVAL, "bwd workspace too small");
  const int64_t sort_bytes = [&] { int64_t p2 = 1; while (p2 < d.cap) p2 <<= 1; return p2 * 4; }();
  if (sort_bytes > 227 * 1024) return fail(PRISM_EINVAL, "too many blocks per head for the backward");
  cudaStream_t st = as_stream(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *delta = reinterpret_cast<float *>(ws + w.delta);
  float *lse2 = reinterpret_cast<float *>(ws + w.lse2);
  int32_t *ccnt = reinterpret_cast<int32_t *>(ws + w.ccnt);
  int32_t *col_ptr = reinterpret_cast<int32_t *>(ws + w.col_ptr);
  int32_t *fill = reinterpret_cast<int32_t *>(ws + w.fill);
  long long *part = reinterpret_cast<long long *>(ws + w.part);
  int32_t *row_idx = reinterpret_cast<int32_t *>(ws + w.row_idx);
  auto O = static_cast<const __nv_bfloat16 *>(o), dO = static_cast<const __nv_bfloat16 *>(dout);
  auto Ores = static_cast<const __nv_bfloat16 *>(o_res);
  if (o_res && !aligned16(o_res)) return fail(PRISM_EINVAL, "bwd: o_res must be 16-byte aligned");
  const int64_t rows = (int64_t)d.heads * d.N;
  const bool tc_path = d.D == 128 && g_attn_backend == 0;
  float *stat_inv = reinterpret_cast<float *>(ws + w.stat_inv);
  uint32_t *amax = reinterpret_cast<uint32_t *>(ws + w.amax);
  uint8_t *f16 = ws + w.f16;
  const size_t tensor_bytes = (size_t)rows * 128 * 2;
  if (tc_path) {
    // per-head maxima of V and dO and their scaled fp16 copies, then D and the P factors
    Tensors2 t2;
    const void *srcs[2] = {v, dout};
    for (int z = 0; z < 2; ++z) {
      t2.src[z] = static_cast<const uint4 *>(srcs[z]);
      t2.dst[z] = reinterpret_cast<uint4 *>(f16 + z * tensor_bytes);
    }
    const int64_t words = d.N * 16;   // 16-byte words per head
    const unsigned gx = (unsigned)std::max<int64_t>(1, std::min<int64_t>((words + 1023) / 1024, (148 * 8 + d.heads - 1) / d.heads));
    if (cudaMemsetAsync(amax, 0, (size_t)d.heads * 2 * 4, st) != cudaSuccess)
      return fail(PRISM_ECUDA, "cudaMemsetAsync failed");
    PRISM_TRACED("head_absmax2_kernel", st, head_absmax2_kernel<<<dim3(gx, d.heads, 2), 256, 0, st>>>(t2, words, d.heads, amax));
    PRISM_TRACED("to_f16x2_kernel", st, to_f16x2_kernel<<<dim3(gx, d.heads, 2), 256, 0, st>>>(t2, words, d.heads, amax));
    PRISM_TRACED("bwd_stats_tc_kernel", st, bwd_stats_tc_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
        O, Ores, dO, lse, rows, delta, lse2, stat_inv));
    cudaMemsetAsync(stat_inv + rows, 0, 128 * 4, st);
  } else if (d.D == 128) {
    PRISM_TRACED("bwd_delta_kernel", st, bwd_delta_kernel<128><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(O, Ores, dO, lse, rows, delta, lse2));
  } else {
    PRISM_TRACED("bwd_delta_kernel", st, bwd_delta_kernel<64><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(O, Ores, dO, lse, rows, delta, lse2));
  }
  cudaMemsetAsync(delta + rows, 0, 128 * 4, st);
  cudaMemsetAsync(lse2 + rows, 0, 128 * 4, st);
  cudaMemsetAsync(ccnt, 0, w.R * 4, st);
  cudaMemsetAsync(fill, 0, w.R * 4, st);
  dim3 rgrid((unsigned)d.cap, d.heads);
  PRISM_TRACED("csc_count_kernel", st, csc_count_kernel<<<rgrid, 256, 0, st>>>(row_ptr, col, d.cap, nblk, ccnt));
  // column counts -> column pointers (their total equals the selection's nnz)
  int64_t *tot = reinterpret_cast<int64_t *>(ws + w.tot);
  rc = launch_scan(ccnt, w.R, part, w.nchunk, col_capacity, col_ptr, tot, st);
  if (rc) return rc;
  PRISM_TRACED("csc_fill_kernel", st, csc_fill_kernel<<<rgrid, 256, 0, st>>>(row_ptr, col, d.cap, nblk, col_ptr, fill, row_idx));
  cudaFuncSetAttribute(csc_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sort_bytes);
  PRISM_TRACED("csc_sort_kernel", st, csc_sort_kernel<<<rgrid, 512, sort_bytes, st>>>(col_ptr, d.cap, nblk, row_idx));
  PRISM_CUDA_CHECK_LAUNCH();
  dim3 grid((unsigned)(d.N / 64), d.heads);
  auto Q = static_cast<const __nv_bfloat16 *>(q), K = static_cast<const __nv_bfloat16 *>(k),
       Vv = static_cast<const __nv_bfloat16 *>(v);
  const float scale = eff_scale(p);
  if (tc_path) {
    CUtensorMap tq, tk, tv, to;
    const uint64_t nrows = (uint64_t)rows;
    if (!make_tile_map(&tq, q, nrows) || !make_tile_map(&tk, k, nrows) ||
        !make_tile_map(&tv, f16, nrows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_tile_map(&to, f16 + tensor_bytes, nrows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
      return fail(PRISM_ECUDA, "cuTensorMapEncodeTiled failed");
    TcBwdArgs a;
    a.blocks = blocks;
    a.zone_blk_base = zone_blk_base;
    a.col_ptr = col_ptr;
    a.row_idx = row_idx;
    a.stat_m = lse2;
    a.stat_inv = stat_inv;
    a.delta_pad = delta;
    a.amax = amax;
    a.heads = d.heads;
    a.N = d.N;
    a.cap = d.cap;
    a.scale = scale;
    a.scale_log2 = scale * kLog2e;
    a.dk = static_cast<__nv_bfloat16 *>(dk);
    a.dv = static_cast<__nv_bfloat16 *>(dv);
    a.wait_limit = g_wait_limit ? g_wait_limit : kDefaultWaitLimit;
    a.debug_stall = g_debug_stall;
    dim3 tgrid((unsigned)(d.Z * 8), d.heads);
    float *dqacc = reinterpret_cast<float *>(ws + w.dqacc);
    if (cudaMemsetAsync(dqacc, 0, (size_t)rows * 128 * 4, st) != cudaSuccess)
      return fail(PRISM_ECUDA, "cudaMemsetAsync failed");
    cudaFuncSetAttribute(bsa_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFbSmemBytes);
    PRISM_TRACED("bsa_bwd_tc_kernel", st, bsa_bwd_tc_kernel<<<tgrid, kFbThreads, kFbSmemBytes, st>>>(tq, tk, tv, to, a, dqacc));
    PRISM_TRACED("dq_convert_kernel", st, dq_convert_kernel<<<dim3((unsigned)(d.N / 64), d.heads), 256, 0, st>>>(
        dqacc, d.N, scale, static_cast<__nv_bfloat16 *>(dq)));
  } else if (d.D == 128)
    rc = launch_bwd_attn<128>(d, grid, st, Q, K, Vv, dO, lse, delta, blocks, zone_blk_base, row_ptr, col, col_ptr,
                         row_idx, scale, static_cast<__nv_bfloat16 *>(dq), static_cast<__nv_bfloat16 *>(dk),
                         static_cast<__nv_bfloat16 *>(dv));
  else
    rc = launch_bwd_attn<64>(d, grid, st, Q, K, Vv, dO, lse, delta, blocks, zone_blk_base, row_ptr, col, col_ptr,
                        row_idx, scale, static_cast<__nv_bfloat16 *>(dq), static_cast<__nv_bfloat16 *>(dk),
                        static_cast<__nv_bfloat16 *>(dv));
  if (rc) return rc;
  PRISM_CUDA_CHECK_LAUNCH();
  return PRISM_OK;
}

}  // extern "C"
