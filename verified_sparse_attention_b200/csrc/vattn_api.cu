// Host side of the C ABI declared in include/vattn.h: argument checks,
// workspace, template dispatch and the launch sequence of one decode step.
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <type_traits>
#include <vector>

#include "vattn.h"
#include "vattn_kernels.cuh"

using vattn::DevParams;
using vattn::UnitInfo;

struct vattn_ctx {
  vattn_config cfg;
  int device = 0;
  int num_sms = 0;
  int G = 1;
  int units_max = 0;
  int score_grid = 0;
  bool score_tma = false;   // contiguous cache: the bulk-copy score pass
  size_t score_smem = 0;
  int gather_grid = 0;     // CTAs of each gather launch
  int CD = 0, CS = 0;      // record producers (warps) of the det/dense and sample gathers
  size_t gather_smem = 0;   // gathers (all modes)
  int gather_threads = 0;
  int draw_splits = 1;
  size_t ws_bytes = 0;
  void* ws = nullptr;
  // carved workspace
  UnitInfo* info = nullptr;
  float* qbar = nullptr;
  float* qsel = nullptr;
  int* dims = nullptr;
  unsigned* ordk = nullptr;
  unsigned* hist = nullptr;
  float* pscore = nullptr;
  int* num_need = nullptr;
  long long* prefix = nullptr;
  unsigned* gcnt = nullptr;
  long long* pre_det = nullptr;
  long long* pre_samp = nullptr;
  float* rec_det = nullptr;
  float* rec_samp = nullptr;
  unsigned* err = nullptr;
  // state
  int last_status = VATTN_OK;
  int last_launches = 0;
  double cached_delta = -1.0;
  double cached_z = 0.0;
  // timing of the score pass
  int timing = 0;            // period (0: off)
  long long timing_calls = 0;
  std::vector<cudaEvent_t> ev_start, ev_stop;
  size_t ev_used = 0;
};

namespace {

// z_{1-delta/2}: 200 bisection steps on [0, 40] of the upper normal tail
// 0.5 * erfc(z / sqrt 2) against delta / 2.
double normal_upper_quantile(double delta) {
  double lo = 0.0, hi = 40.0;
  const double target = 0.5 * delta;
  for (int it = 0; it < 200; it++) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * erfc(mid * 0.70710678118654752440) > target)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The driver's tensor-map encoder, reached through the runtime (the library
// does not link the driver library itself).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Row maps of the K and V caches for the gathers: a 2-D [rows][d] view with
// rows = num_pages * Hkv * page_size, one-row boxes of all d columns.
int encode_row_maps(const vattn_config& c, const void* k, const void* v, int num_pages, DevParams* P) {
  const unsigned long long rows =
      static_cast<unsigned long long>(num_pages) * c.num_kv_heads * static_cast<unsigned long long>(c.page_size);
  if (rows > 0x7FFFFFFFull) return VATTN_EINVAL;  // row coordinates are 32-bit
  const EncodeTiledFn fn = encode_tiled();
  if (!fn) return VATTN_ECUDA;
  const cuuint64_t esz = c.dtype == VATTN_BF16 ? 2 : 4;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(c.head_dim), rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(c.head_dim) * esz};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(c.head_dim), 1u};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUtensorMapDataType dt =
      c.dtype == VATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  for (int i = 0; i < 2; i++) {
    const CUresult r = fn(i ? &P->tmv : &P->tmk, dt, 2, const_cast<void*>(i ? v : k), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return VATTN_ECUDA;
  }
  if (c.dtype == VATTN_BF16) {  // the tensor-core gathers' swizzled half-row boxes
    const cuuint32_t hbox[2] = {64u, 1u};
    for (int i = 0; i < 2; i++) {
      const CUresult r = fn(i ? &P->tmv_sw : &P->tmk_sw, dt, 2, const_cast<void*>(i ? v : k), dims, strides, hbox,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return VATTN_ECUDA;
    }
  }
  return VATTN_OK;
}

// ---------------------------------------------------------------- dispatch
struct Kernels {
  void (*prep)(DevParams);
  void (*score_exact)(DevParams);
  void (*score_loki)(DevParams);
  void (*score_sparq)(DevParams);
  void (*score_exact_tma)(DevParams);  // contiguous caches
  void (*score_loki_tma)(DevParams);
  size_t score_tma_smem, score_loki_tma_smem;
  void (*det)(DevParams);
  void (*sample)(DevParams);
  void (*dense)(DevParams);
  void (*det_host)(DevParams);     // the gathers for caches in host memory
  void (*sample_host)(DevParams);
  void (*dense_host)(DevParams);
  void (*sample_tc)(DevParams);    // tensor-core sample and dense gathers (bf16, device caches)
  void (*dense_tc)(DevParams);
  size_t tc_smem;
  void (*budget)(DevParams);
  void (*numstats)(DevParams);
  void (*combine_sample)(DevParams);
  void (*combine_dense)(DevParams);
  size_t gather_smem;
  int gather_threads;
};

template <typename T, int D, int G>
Kernels kernels_for() {
  Kernels k;
  k.prep = vattn::k_prep<T, D, G>;
  k.score_exact = vattn::k_score_rows<T, D>;
  k.score_loki = vattn::k_score_rows<T, 32>;
  k.score_exact_tma = vattn::k_score_tma<T, D>;
  k.score_loki_tma = vattn::k_score_tma<T, 32>;
  k.score_tma_smem = vattn::ScoreShape<T, D>::SMEM;
  k.score_loki_tma_smem = vattn::ScoreShape<T, 32>::SMEM;
  k.score_sparq = vattn::k_score_sparq<T, D>;
  k.det = vattn::k_gather<T, D, G, vattn::kModeDet>;
  k.sample = vattn::k_gather<T, D, G, vattn::kModeSample>;
  k.dense = vattn::k_gather<T, D, G, vattn::kModeDense>;
  k.det_host = vattn::k_gather<T, D, G, vattn::kModeDet, true>;
  k.sample_host = vattn::k_gather<T, D, G, vattn::kModeSample, true>;
  k.dense_host = vattn::k_gather<T, D, G, vattn::kModeDense, true>;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    k.sample_tc = vattn::k_gather_tc<D, G, vattn::kModeSample>;
    k.dense_tc = vattn::k_gather_tc<D, G, vattn::kModeDense>;
    k.tc_smem = vattn::TcShape<D, G>::SMEM;
  } else {
    k.sample_tc = k.dense_tc = nullptr;
    k.tc_smem = 0;
  }
  k.budget = vattn::k_budget<D, G>;
  k.numstats = vattn::k_numstats<T, D, G>;
  k.combine_sample = vattn::k_combine<D, G, vattn::kModeSample>;
  k.combine_dense = vattn::k_combine<D, G, vattn::kModeDense>;
  k.gather_smem = vattn::GatherShape<T, D, G>::SMEM;
  k.gather_threads = vattn::GatherShape<T, D, G>::NW * 32;
  return k;
}

template <typename T, int D>
bool pick_g(int G, Kernels* k) {
  switch (G) {
    case 1: *k = kernels_for<T, D, 1>(); return true;
    case 2: *k = kernels_for<T, D, 2>(); return true;
    case 4: *k = kernels_for<T, D, 4>(); return true;
    case 8: *k = kernels_for<T, D, 8>(); return true;
    default: return false;
  }
}

bool pick(const vattn_config& c, int G, Kernels* k) {
  if (c.dtype == VATTN_BF16) {
    if (c.head_dim == 128) return pick_g<__nv_bfloat16, 128>(G, k);
    if (c.head_dim == 64) return pick_g<__nv_bfloat16, 64>(G, k);
  } else if (c.dtype == VATTN_FP32) {
    if (c.head_dim == 128) return pick_g<float, 128>(G, k);
    if (c.head_dim == 64) return pick_g<float, 64>(G, k);
  }
  return false;
}

int check_config(const vattn_config* c) {
  if (!c) return VATTN_EINVAL;
  if (c->num_kv_heads < 1 || c->num_q_heads < 1 || c->num_q_heads % c->num_kv_heads) return VATTN_EINVAL;
  const int G = c->num_q_heads / c->num_kv_heads;
  if (!(G == 1 || G == 2 || G == 4 || G == 8)) return VATTN_EINVAL;
  if (!(c->head_dim == 64 || c->head_dim == 128)) return VATTN_EINVAL;
  if (!(c->dtype == VATTN_FP32 || c->dtype == VATTN_BF16)) return VATTN_EINVAL;
  if (c->page_size < 16 || c->page_size % 16) return VATTN_EINVAL;
  if (c->max_batch < 1 || c->max_ctx < 1 || c->max_ctx > (1 << 24)) return VATTN_EINVAL;
  if (c->proxy == VATTN_SPARQ) {
    if (c->proxy_rank < 1 || c->proxy_rank > c->head_dim) return VATTN_EINVAL;
  } else if (c->proxy == VATTN_LOKI) {
    if (c->proxy_rank != 32) return VATTN_EINVAL;
  } else if (c->proxy != VATTN_EXACT) {
    return VATTN_EINVAL;
  }
  if (c->kv_location != VATTN_KV_DEVICE && c->kv_location != VATTN_KV_HOST) return VATTN_EINVAL;
  return VATTN_OK;
}

// Device address of a cache in page-locked host memory (nullptr if `p` is not
// such memory).
const void* host_cache_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
  return static_cast<const char*>(a.devicePointer) +
         (static_cast<const char*>(p) - static_cast<const char*>(a.hostPointer ? a.hostPointer : p));
}

// The caches as the kernels address them (host-resident caches mapped to
// their device addresses); VATTN_EINVAL if a host-resident cache is not
// page-locked.
int cache_ptrs(const vattn_config& c, const void** k, const void** v) {
  if (c.kv_location != VATTN_KV_HOST) return VATTN_OK;
  const void* dk = host_cache_device_ptr(*k);
  const void* dv = host_cache_device_ptr(*v);
  if (!dk || !dv) return VATTN_EINVAL;
  *k = dk;
  *v = dv;
  return VATTN_OK;
}

void fill_common(const vattn_ctx* ctx, DevParams* P, int batch) {
  memset(P, 0, sizeof(*P));
  const vattn_config& c = ctx->cfg;
  P->Hq = c.num_q_heads;
  P->Hkv = c.num_kv_heads;
  P->G = ctx->G;
  P->D = c.head_dim;
  P->pps = (c.max_ctx + c.page_size - 1) / c.page_size;
  P->ps = c.page_size;
  P->ps_magic = ~0ull / static_cast<unsigned long long>(c.page_size) + 1ull;
  P->max_ctx = c.max_ctx;
  P->batch = batch;
  P->units = batch * c.num_kv_heads;
  P->proxy = c.proxy;
  P->rank = c.proxy_rank;
  P->kv_host = c.kv_location == VATTN_KV_HOST;
  P->scale = static_cast<float>(1.0 / sqrt(static_cast<double>(c.head_dim)));
  P->info = ctx->info;
  P->qbar = ctx->qbar;
  P->qsel = ctx->qsel;
  P->dims = ctx->dims;
  P->ordk = ctx->ordk;
  P->hist = ctx->hist;
  P->pscore = ctx->pscore;
  P->num_need = ctx->num_need;
  P->prefix = ctx->prefix;
  P->gcnt = ctx->gcnt;
  P->pre_det = ctx->pre_det;
  P->pre_samp = ctx->pre_samp;
  P->rec_det = ctx->rec_det;
  P->rec_samp = ctx->rec_samp;
  P->CD = ctx->CD;
  P->CS = ctx->CS;
  P->err = ctx->err;
}

// Launch with programmatic dependent launch: the kernel may be scheduled while
// its predecessor on the stream drains; it waits (griddepcontrol.wait) before
// reading the predecessor's results.
void launch(void (*kern)(DevParams), dim3 grid, dim3 block, size_t smem, cudaStream_t st, const DevParams& P,
            int* count) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kern, P);
  (*count)++;
}

// Threads of a combine CTA (one per unit and head): sixteen warps while the
// CTAs fit one wave at two per SM, else eight.
int comb_threads(const vattn_ctx* ctx, int units) {
  const long long ctas = static_cast<long long>(units) * ctx->G;
  return (ctas <= 2LL * ctx->num_sms ? vattn::kCombWarps : vattn::kCombWarps / 2) * 32;
}

int finish(vattn_ctx* ctx, int launches) {
  ctx->last_launches = launches;
  const cudaError_t e = cudaGetLastError();
  ctx->last_status = e == cudaSuccess ? VATTN_OK : VATTN_ECUDA;
  return ctx->last_status;
}

}  // namespace

extern "C" {

const char* vattn_strerror(int code) {
  switch (code) {
    case VATTN_OK: return "ok";
    case VATTN_EINVAL: return "invalid argument";
    case VATTN_ENOMEM: return "device workspace allocation failed";
    case VATTN_ECUDA: return "CUDA call or kernel launch failed";
    case VATTN_ESCRATCH: return "call needs more than the fixed 8 MiB scratch array of vattn_dense_decode_static";
    default: return "unknown code";
  }
}

int vattn_create(vattn_ctx** out, const vattn_config* cfg) {
  if (!out) return VATTN_EINVAL;
  *out = nullptr;
  if (check_config(cfg) != VATTN_OK) return VATTN_EINVAL;
  vattn_ctx* ctx = new vattn_ctx();
  ctx->cfg = *cfg;
  ctx->G = cfg->num_q_heads / cfg->num_kv_heads;
  Kernels K;
  if (!pick(ctx->cfg, ctx->G, &K)) {
    delete ctx;
    return VATTN_EINVAL;
  }
  if (cudaGetDevice(&ctx->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device) != cudaSuccess) {
    delete ctx;
    return VATTN_ECUDA;
  }
  const int D = cfg->head_dim, G = ctx->G;
  const size_t U = static_cast<size_t>(cfg->max_batch) * cfg->num_kv_heads;
  ctx->units_max = static_cast<int>(U);

  // grid sizes: the score pass and the gathers run one wave of resident CTAs
  void (*score)(DevParams) = cfg->proxy == VATTN_SPARQ ? K.score_sparq
                             : cfg->proxy == VATTN_LOKI ? K.score_loki : K.score_exact;
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, score, 256, 0);
  ctx->score_grid = (occ < 1 ? 1 : occ) * ctx->num_sms;
  // the bulk-copy score pass streams a contiguous cache in device memory (the
  // proxy cache for Loki, K itself in exact mode)
  if (cfg->page_size >= cfg->max_ctx && cfg->proxy != VATTN_SPARQ &&
      (cfg->proxy == VATTN_LOKI || cfg->kv_location == VATTN_KV_DEVICE)) {
    void (*tma)(DevParams) = cfg->proxy == VATTN_LOKI ? K.score_loki_tma : K.score_exact_tma;
    const size_t smem = cfg->proxy == VATTN_LOKI ? K.score_loki_tma_smem : K.score_tma_smem;
    if (cudaFuncSetAttribute(tma, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) ==
        cudaSuccess) {
      ctx->score_tma = true;
      ctx->score_smem = smem;
    }
    cudaGetLastError();
  }
  ctx->gather_smem = K.gather_smem;
  ctx->gather_threads = K.gather_threads;
  for (auto fn : {K.det, K.sample, K.dense, K.det_host, K.sample_host, K.dense_host})
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(ctx->gather_smem));
  for (auto fn : {K.sample_tc, K.dense_tc})
    if (fn) cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(K.tc_smem));
  cudaFuncSetAttribute(K.numstats, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(vattn::kNumSmem));
  int gocc = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&gocc, K.sample, K.gather_threads, ctx->gather_smem);
  if (gocc < 1) gocc = 1;
  ctx->gather_grid = gocc * ctx->num_sms;
  ctx->CD = ctx->CS = ctx->gather_grid * (K.gather_threads / 32);
  ctx->draw_splits = std::max(1, (2 * ctx->num_sms + static_cast<int>(U) - 1) / static_cast<int>(U));
  if (cudaGetLastError() != cudaSuccess) {
    delete ctx;
    return VATTN_ECUDA;
  }

  const size_t REC = static_cast<size_t>(G) * (2 + D);
  const size_t sz_info = align256(U * sizeof(UnitInfo));
  const size_t sz_vec = align256(U * D * sizeof(float));
  const size_t sz_ordk = align256(U * cfg->max_ctx * sizeof(unsigned));
  const size_t sz_hist = align256(U * vattn::kHist1 * sizeof(unsigned));
  const size_t sz_ps = align256(U * cfg->max_ctx * G * sizeof(float));
  const size_t sz_nneed = align256(U * G * sizeof(int));
  const size_t sz_pre = align256((U + 1) * sizeof(long long));
  const size_t sz_gcnt = 256;
  const size_t sz_spre = align256((2 * U + 1) * sizeof(long long));
  const size_t sz_rdet = align256((ctx->CD + 2 * U) * REC * sizeof(float));
  const size_t sz_rsmp = align256((ctx->CS + 2 * U) * REC * sizeof(float));
  const size_t sz_err = 256;
  ctx->ws_bytes = sz_info + 3 * sz_vec + sz_ordk + sz_hist + sz_ps + sz_nneed + sz_pre + sz_gcnt +
                  2 * sz_spre + sz_rdet + sz_rsmp + sz_err;
  if (cudaMalloc(&ctx->ws, ctx->ws_bytes) != cudaSuccess) {
    cudaGetLastError();
    delete ctx;
    return VATTN_ENOMEM;
  }
  char* p = static_cast<char*>(ctx->ws);
  ctx->info = reinterpret_cast<UnitInfo*>(p); p += sz_info;
  ctx->qbar = reinterpret_cast<float*>(p); p += sz_vec;
  ctx->qsel = reinterpret_cast<float*>(p); p += sz_vec;
  ctx->dims = reinterpret_cast<int*>(p); p += sz_vec;
  ctx->ordk = reinterpret_cast<unsigned*>(p); p += sz_ordk;
  ctx->hist = reinterpret_cast<unsigned*>(p); p += sz_hist;
  ctx->pscore = reinterpret_cast<float*>(p); p += sz_ps;
  ctx->num_need = reinterpret_cast<int*>(p); p += sz_nneed;
  ctx->prefix = reinterpret_cast<long long*>(p); p += sz_pre;
  ctx->gcnt = reinterpret_cast<unsigned*>(p); p += sz_gcnt;
  ctx->pre_det = reinterpret_cast<long long*>(p); p += sz_spre;
  ctx->pre_samp = reinterpret_cast<long long*>(p); p += sz_spre;
  ctx->rec_det = reinterpret_cast<float*>(p); p += sz_rdet;
  ctx->rec_samp = reinterpret_cast<float*>(p); p += sz_rsmp;
  ctx->err = reinterpret_cast<unsigned*>(p);
  if (cudaMemset(ctx->ws, 0, ctx->ws_bytes) != cudaSuccess) {
    cudaFree(ctx->ws);
    delete ctx;
    return VATTN_ECUDA;
  }
  // the top-k selection (k_topk, two block sizes)
  if (cudaFuncSetAttribute(vattn::k_topk<vattn::kTopkThreads>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(vattn::kTopkKernelSmem)) != cudaSuccess ||
      cudaFuncSetAttribute(vattn::k_topk<vattn::kTopkThreadsFew>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(vattn::kTopkKernelSmem)) != cudaSuccess) {
    cudaFree(ctx->ws);
    delete ctx;
    return VATTN_ECUDA;
  }
  *out = ctx;
  return VATTN_OK;
}

void vattn_destroy(vattn_ctx* ctx) {
  if (!ctx) return;
  for (auto e : ctx->ev_start) cudaEventDestroy(e);
  for (auto e : ctx->ev_stop) cudaEventDestroy(e);
  if (ctx->ws) cudaFree(ctx->ws);
  delete ctx;
}

size_t vattn_workspace_bytes(const vattn_ctx* ctx) { return ctx ? ctx->ws_bytes : 0; }

int vattn_last_launch_count(const vattn_ctx* ctx) { return ctx ? ctx->last_launches : 0; }

int vattn_set_timing(vattn_ctx* ctx, int period) {
  if (!ctx || period < 0) return VATTN_EINVAL;
  ctx->timing = period;
  ctx->timing_calls = 0;
  return VATTN_OK;
}

int vattn_score_pass_ms(vattn_ctx* ctx, double* total_ms, int* count, int reset) {
  if (!ctx || !total_ms || !count) return VATTN_EINVAL;
  double tot = 0.0;
  for (size_t i = 0; i < ctx->ev_used; i++) {
    if (cudaEventSynchronize(ctx->ev_stop[i]) != cudaSuccess) return VATTN_ECUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, ctx->ev_start[i], ctx->ev_stop[i]) != cudaSuccess) return VATTN_ECUDA;
    tot += ms;
  }
  *total_ms = tot;
  *count = static_cast<int>(ctx->ev_used);
  if (reset) ctx->ev_used = 0;
  return VATTN_OK;
}

int vattn_last_error(vattn_ctx* ctx, int sync) {
  if (!ctx) return VATTN_EINVAL;
  if (!sync) return ctx->last_status;
  if (cudaDeviceSynchronize() != cudaSuccess) return VATTN_ECUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, ctx->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return VATTN_ECUDA;
  if (cudaMemset(ctx->err, 0, sizeof(unsigned)) != cudaSuccess) return VATTN_ECUDA;
  return static_cast<int>(v);
}

int vattn_check_bounded_wait(vattn_ctx* ctx, int tries, void* stream) {
  if (!ctx || tries < 1 || tries > vattn::kWaitTries) return VATTN_EINVAL;
  vattn::k_wait_check<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ctx->err, tries);
  return cudaGetLastError() == cudaSuccess ? VATTN_OK : VATTN_ECUDA;
}

int vattn_decode(vattn_ctx* ctx, const void* q, const void* k_cache, const void* v_cache,
                 const int32_t* page_table, const int32_t* seq_lens, int batch,
                 const vattn_params* prm, float* out, int32_t* sel_idx, int32_t* sel_count,
                 int32_t* budgets, int32_t* head_need, void* stream) {
  if (!ctx) return VATTN_EINVAL;
  ctx->last_status = VATTN_EINVAL;
  const vattn_config& c = ctx->cfg;
  if (!prm || !q || !k_cache || !v_cache || !page_table || !seq_lens || !out || !sel_idx ||
      !sel_count || !budgets || !head_need)
    return VATTN_EINVAL;
  if (batch < 0 || batch > c.max_batch) return VATTN_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return VATTN_EINVAL;
  if (prm->sinks < 0 || prm->window < 0 || prm->topk_abs < 0 || prm->topk_den < 0 ||
      prm->topk_num < 0 || prm->pilot_num < 0 || prm->pilot_den < 0)
    return VATTN_EINVAL;
  if (prm->topk_den > 0 && prm->topk_num > prm->topk_den) return VATTN_EINVAL;
  if (prm->pilot_den > 0 && prm->pilot_num > prm->pilot_den) return VATTN_EINVAL;
  if (prm->pilot_min < 2 || prm->pilot_min > (1 << 24)) return VATTN_EINVAL;
  if (!(prm->eps > 0.0f) || !isfinite(prm->eps)) return VATTN_EINVAL;
  if (!(prm->delta > 0.0f && prm->delta < 1.0f)) return VATTN_EINVAL;
  if (prm->num_pages < 1) return VATTN_EINVAL;
  if (prm->guarantee != VATTN_GUARANTEE_DENOMINATOR && prm->guarantee != VATTN_GUARANTEE_OUTPUT)
    return VATTN_EINVAL;
  if (prm->topp_den < 0 || prm->topp_num < 0 || prm->topp_num > prm->topp_den) return VATTN_EINVAL;
  if (prm->batch_offset < 0 || prm->head_offset < 0) return VATTN_EINVAL;
  if (c.proxy == VATTN_SPARQ && (!prm->k_t_cache || !aligned16(prm->k_t_cache))) return VATTN_EINVAL;
  if (c.proxy == VATTN_LOKI && (!prm->k_proj_cache || !prm->proj_basis || !aligned16(prm->k_proj_cache)))
    return VATTN_EINVAL;
  Kernels K;
  if (!pick(c, ctx->G, &K)) return VATTN_EINVAL;
  if (batch == 0) {
    ctx->last_launches = 0;
    return ctx->last_status = VATTN_OK;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  DevParams P;
  fill_common(ctx, &P, batch);
  P.sinks = prm->sinks;
  P.window = prm->window;
  P.topk_abs = prm->topk_abs;
  P.topk_num = prm->topk_num;
  P.topk_den = prm->topk_den;
  P.pilot_min = prm->pilot_min;
  P.pilot_num = prm->pilot_num;
  P.pilot_den = prm->pilot_den;
  P.eps = prm->eps;
  if (static_cast<double>(prm->delta) != ctx->cached_delta) {
    ctx->cached_delta = static_cast<double>(prm->delta);
    ctx->cached_z = normal_upper_quantile(ctx->cached_delta);
  }
  P.z = ctx->cached_z;
  P.seed = prm->seed;
  P.num_pages = prm->num_pages;
  P.guarantee = prm->guarantee == VATTN_GUARANTEE_OUTPUT;
  P.topp_num = prm->topp_num;
  P.topp_den = prm->topp_den;
  P.batch_offset = prm->batch_offset;
  P.head_offset = prm->head_offset;
  if (const int rc = cache_ptrs(c, &k_cache, &v_cache)) return ctx->last_status = rc;
  // row maps for the gathers' tensor copies (host-resident caches use plain loads)
  if (!P.kv_host)
    if (const int rc = encode_row_maps(c, k_cache, v_cache, prm->num_pages, &P)) return ctx->last_status = rc;
  P.q = q;
  P.k = k_cache;
  P.v = v_cache;
  P.kt = prm->k_t_cache;
  P.kp = prm->k_proj_cache;
  P.basis = prm->proj_basis;
  P.page_table = page_table;
  P.seq_lens = seq_lens;
  P.out = out;
  P.sel = sel_idx;
  P.sel_count = sel_count;
  P.budgets = budgets;
  P.head_need = head_need;
  P.dense = 0;

  int launches = 0;
  launch(K.prep, dim3(P.units + 1), dim3(128), 0, st, P, &launches);
  void (*score)(DevParams) = c.proxy == VATTN_SPARQ ? K.score_sparq
                             : c.proxy == VATTN_LOKI ? K.score_loki : K.score_exact;
  const bool timed = ctx->timing > 0 && (ctx->timing_calls++ % ctx->timing) == 0;
  if (timed) {
    if (ctx->ev_used == ctx->ev_start.size()) {
      cudaEvent_t a, b;
      cudaEventCreate(&a);
      cudaEventCreate(&b);
      ctx->ev_start.push_back(a);
      ctx->ev_stop.push_back(b);
    }
    cudaEventRecord(ctx->ev_start[ctx->ev_used], st);
  }
  if (ctx->score_tma)
    launch(c.proxy == VATTN_LOKI ? K.score_loki_tma : K.score_exact_tma, dim3(ctx->num_sms), dim3(256),
           ctx->score_smem, st, P, &launches);
  else
    launch(score, dim3(ctx->score_grid), dim3(256), 0, st, P, &launches);
  if (timed) {
    cudaEventRecord(ctx->ev_stop[ctx->ev_used], st);
    ctx->ev_used++;
  }
  // top-p: each unit's top-k size from the mass of its ranking scores
  if (P.topp_den > 0) launch(vattn::k_topp, dim3(P.units), dim3(vattn::kToppThreads), 0, st, P, &launches);
  // top-k select and pilot draws, one CTA per unit
  if (P.units <= ctx->num_sms)
    launch(vattn::k_topk<vattn::kTopkThreadsFew>, dim3(P.units), dim3(vattn::kTopkThreadsFew),
           vattn::kTopkKernelSmem, st, P, &launches);
  else
    launch(vattn::k_topk<vattn::kTopkThreads>, dim3(P.units), dim3(vattn::kTopkThreads), vattn::kTopkKernelSmem,
           st, P, &launches);
  launch(P.kv_host ? K.det_host : K.det, dim3(ctx->gather_grid), dim3(ctx->gather_threads), ctx->gather_smem, st, P, &launches);
  if (P.guarantee)
    launch(K.numstats, dim3(P.units, (ctx->G * c.head_dim + vattn::kNumThreads - 1) / vattn::kNumThreads),
           dim3(vattn::kNumThreads), vattn::kNumSmem, st, P, &launches);
  launch(K.budget, dim3(P.units), dim3(vattn::kBudgetThreads), 0, st, P, &launches);
  launch(vattn::k_draws, dim3(P.units, ctx->draw_splits * 4), dim3(128), 0, st, P, &launches);
  if (!P.kv_host && K.sample_tc)
    launch(K.sample_tc, dim3(ctx->gather_grid), dim3(ctx->gather_threads), K.tc_smem, st, P, &launches);
  else
    launch(P.kv_host ? K.sample_host : K.sample, dim3(ctx->gather_grid), dim3(ctx->gather_threads), ctx->gather_smem,
           st, P, &launches);
  launch(K.combine_sample, dim3(P.units, ctx->G), dim3(comb_threads(ctx, P.units)), 0, st, P, &launches);
  return finish(ctx, launches);
}

int vattn_dense_decode(vattn_ctx* ctx, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* page_table, const int32_t* seq_lens, int batch, int num_pages,
                       float* out, void* stream) {
  if (!ctx) return VATTN_EINVAL;
  ctx->last_status = VATTN_EINVAL;
  const vattn_config& c = ctx->cfg;
  if (!q || !k_cache || !v_cache || !page_table || !seq_lens || !out) return VATTN_EINVAL;
  if (batch < 0 || batch > c.max_batch || num_pages < 1) return VATTN_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return VATTN_EINVAL;
  Kernels K;
  if (!pick(c, ctx->G, &K)) return VATTN_EINVAL;
  if (batch == 0) {
    ctx->last_launches = 0;
    return ctx->last_status = VATTN_OK;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevParams P;
  fill_common(ctx, &P, batch);
  // no selection: sinks cover everything, so every unit is a deterministic
  // set of all positions with no middle to rank
  P.sinks = c.max_ctx;
  P.window = 0;
  P.pilot_min = 2;
  P.eps = 1.0f;
  P.num_pages = num_pages;
  if (const int rc = cache_ptrs(c, &k_cache, &v_cache)) return ctx->last_status = rc;
  if (!P.kv_host)
    if (const int rc = encode_row_maps(c, k_cache, v_cache, num_pages, &P)) return ctx->last_status = rc;
  P.proxy = VATTN_EXACT;
  P.q = q;
  P.k = k_cache;
  P.v = v_cache;
  P.page_table = page_table;
  P.seq_lens = seq_lens;
  P.out = out;
  P.dense = 1;
  // prep only validates and fills the unit state here; its index writes go to
  // the workspace copy of the selection list, never to caller memory
  P.sel = reinterpret_cast<int*>(ctx->ordk);
  int launches = 0;
  launch(K.prep, dim3(P.units + 1), dim3(128), 0, st, P, &launches);
  if (!P.kv_host && K.dense_tc)
    launch(K.dense_tc, dim3(ctx->gather_grid), dim3(ctx->gather_threads), K.tc_smem, st, P, &launches);
  else
    launch(P.kv_host ? K.dense_host : K.dense, dim3(ctx->gather_grid), dim3(ctx->gather_threads), ctx->gather_smem,
           st, P, &launches);
  launch(K.combine_dense, dim3(P.units, ctx->G), dim3(comb_threads(ctx, P.units)), 0, st, P, &launches);
  return finish(ctx, launches);
}

}  // extern "C"
