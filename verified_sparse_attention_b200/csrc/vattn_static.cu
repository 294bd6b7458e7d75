// vattn_dense_decode_static: dense decode attention that allocates nothing.
//
// The other entry points keep their scratch in a context workspace that
// vattn_create allocates. This one needs no context: its only scratch is the
// file-scope device array below, of a fixed size, whose address is looked up
// once per CUDA context (normally once per device; again after a device
// reset). It exists for callers that cannot allocate device memory
// at the point of the call (a server that has handed all free memory to its
// KV-cache pool, code that must not risk the device-wide synchronisation a
// free can cause, or a plug-in that cannot keep a context between calls).
//
// Work split (flash-decoding style, two kernels on the caller's stream):
//   k_dense_split  grid (S, units): CTA (s, u) folds positions
//                  [n*s/S, n*(s+1)/S) of unit u = (sequence b, KV head h)
//                  into one record per query head of the group: the running
//                  max m, the exp sum l and the exp-weighted value sum acc[d];
//   k_dense_merge  grid (units): merges the S records of each head and
//                  writes out = acc / l (0 for an empty sequence).
// Every record a call reads is written earlier in the same call, so nothing
// in the array has to start at zero and the previous call's contents are
// harmless. Two calls that overlap in time on one device (other streams,
// other host threads) share the array and race: order them.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "vattn.h"
#include "vattn_device.cuh"

namespace {

using vattn::Elem;
using vattn::ld_gather;

// Fixed maximum of the array: 8 MiB per device. A call needs at least one
// record of G * (d + 2) floats per (sequence, KV head), i.e.
// batch * Hq * (d + 2) * 4 bytes; larger calls are refused (VATTN_ESCRATCH).
constexpr size_t kStaticScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_dense_scratch[kStaticScratchBytes / sizeof(float)];

struct StaticArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* out;
  float* rec;  // [units][S][G][d + 2] inside the static array
  int Hq, Hkv, pps, ps, max_ctx, num_pages;
  float scale;
};

constexpr int kWarps = 8;

// Row layout of a warp: NC 16-byte chunks per row, one lane per chunk, so a
// warp holds 32 / NC rows at once and UNR such row groups are loaded before
// any is used. A lane's partial dot product is a fused multiply-add chain
// over its chunk; the butterfly over the row's lanes then adds the chunk sums
// pairwise at halving strides.
template <typename T, int D>
struct DenseShape {
  static constexpr int E = Elem<T>::kPer16;
  static constexpr int NC = D / E;
  static constexpr int RPW = 32 / NC;  // rows per warp-wide load
  static constexpr int UNR = 4;
  static constexpr int RB = RPW * UNR;  // rows per warp iteration
};

__device__ __forceinline__ float exp_rel(float x, float m) {
  return m == -INFINITY ? 0.0f : __expf(x - m);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kWarps * 32) k_dense_split(StaticArgs A) {
  using S = DenseShape<T, D>;
  constexpr int E = S::E, NC = S::NC, UNR = S::UNR, RPW = S::RPW, RB = S::RB;
  constexpr int REC = G * (D + 2);
  __shared__ float s_m[kWarps][G], s_l[kWarps][G];
  __shared__ float s_acc[kWarps][G][D];

  const int u = blockIdx.y, sp = blockIdx.x, nsp = gridDim.x;
  const int b = u / A.Hkv, h = u % A.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / NC, c = lane % NC;

  // sequence length and page ids; a bad sequence is treated as empty
  int n = A.seq_lens[b];
  if (n < 0 || n > A.max_ctx) n = 0;
  const int npages = (n + A.ps - 1) / A.ps;
  int bad = 0;
  for (int i = threadIdx.x; i < npages; i += blockDim.x) {
    const int pid = A.page_table[static_cast<size_t>(b) * A.pps + i];
    if (pid < 0 || pid >= A.num_pages) bad = 1;
  }
  if (__syncthreads_or(bad)) n = 0;
  const int j0 = static_cast<int>(static_cast<long long>(n) * sp / nsp);
  const int j1 = static_cast<int>(static_cast<long long>(n) * (sp + 1) / nsp);

  // my chunk of each query head of the group, fp32
  float qv[G][E];
#pragma unroll
  for (int g = 0; g < G; g++)
#pragma unroll
    for (int e = 0; e < E; e++)
      qv[g][e] = Elem<T>::load(A.q, (static_cast<size_t>(b) * A.Hq + h * G + g) * D + c * E + e);

  float m[G], l[G], acc[G][E];
#pragma unroll
  for (int g = 0; g < G; g++) {
    m[g] = -INFINITY;
    l[g] = 0.0f;
#pragma unroll
    for (int e = 0; e < E; e++) acc[g][e] = 0.0f;
  }
  const T* kc = static_cast<const T*>(A.k);
  const T* vc = static_cast<const T*>(A.v);

  // the trip count depends on the warp only, so every shuffle below runs
  // with the whole warp
  for (int base = j0 + warp * RB; base < j1; base += kWarps * RB) {
    uint4 kr[UNR], vr[UNR];
    bool ok[UNR];
#pragma unroll
    for (int k = 0; k < UNR; k++) {
      const int pos = base + k * RPW + grp;
      ok[k] = pos < j1;
      kr[k] = vr[k] = make_uint4(0u, 0u, 0u, 0u);
      if (ok[k]) {
        const int slot = pos / A.ps;
        const size_t page = static_cast<size_t>(A.page_table[static_cast<size_t>(b) * A.pps + slot]);
        const size_t off = ((page * A.Hkv + h) * A.ps + (pos - slot * A.ps)) * D + c * E;
        kr[k] = ld_gather(kc + off);
        vr[k] = ld_gather(vc + off);
      }
    }
    float sc[UNR][G];
#pragma unroll
    for (int k = 0; k < UNR; k++) {
      float kx[E];
      Elem<T>::unpack(kr[k], kx);
#pragma unroll
      for (int g = 0; g < G; g++) {
        float a = 0.0f;
#pragma unroll
        for (int e = 0; e < E; e++) a = __fmaf_rn(qv[g][e], kx[e], a);
#pragma unroll
        for (int o = NC / 2; o >= 1; o >>= 1) a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, o));
        sc[k][g] = ok[k] ? __fmul_rn(a, A.scale) : -INFINITY;
      }
    }
    // online softmax, one rescale per iteration
#pragma unroll
    for (int g = 0; g < G; g++) {
      float bm = sc[0][g];
#pragma unroll
      for (int k = 1; k < UNR; k++) bm = fmaxf(bm, sc[k][g]);
      if (bm > m[g]) {
        const float cf = exp_rel(m[g], bm);
        l[g] *= cf;
#pragma unroll
        for (int e = 0; e < E; e++) acc[g][e] *= cf;
        m[g] = bm;
      }
#pragma unroll
      for (int k = 0; k < UNR; k++) {
        sc[k][g] = sc[k][g] == -INFINITY ? 0.0f : __expf(sc[k][g] - m[g]);
        l[g] += sc[k][g];
      }
    }
#pragma unroll
    for (int k = 0; k < UNR; k++) {
      float vx[E];
      Elem<T>::unpack(vr[k], vx);
#pragma unroll
      for (int g = 0; g < G; g++)
#pragma unroll
        for (int e = 0; e < E; e++) acc[g][e] = fmaf(sc[k][g], vx[e], acc[g][e]);
    }
  }

  // merge the warp's row groups (lanes c, c + NC, ... hold the same chunk)
#pragma unroll
  for (int o = NC; o < 32; o <<= 1) {
#pragma unroll
    for (int g = 0; g < G; g++) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[g], o);
      const float lo = __shfl_xor_sync(0xffffffffu, l[g], o);
      const float M = fmaxf(m[g], mo);
      const float ca = exp_rel(m[g], M), cb = exp_rel(mo, M);
      l[g] = l[g] * ca + lo * cb;
#pragma unroll
      for (int e = 0; e < E; e++) {
        const float ao = __shfl_xor_sync(0xffffffffu, acc[g][e], o);
        acc[g][e] = acc[g][e] * ca + ao * cb;
      }
      m[g] = M;
    }
  }
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
      for (int e = 0; e < E; e++) s_acc[warp][g][c * E + e] = acc[g][e];
    if (c == 0) {
#pragma unroll
      for (int g = 0; g < G; g++) {
        s_m[warp][g] = m[g];
        s_l[warp][g] = l[g];
      }
    }
  }
  __syncthreads();
  // merge the warps into this CTA's records
  float* r = A.rec + (static_cast<size_t>(u) * nsp + sp) * REC;
  for (int x = threadIdx.x; x < G * D; x += blockDim.x) {
    const int g = x / D, d = x % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) M = fmaxf(M, s_m[w][g]);
    float a = 0.0f, ls = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; w++) {
      const float cw = exp_rel(s_m[w][g], M);
      a += s_acc[w][g][d] * cw;
      ls += s_l[w][g] * cw;
    }
    r[g * (D + 2) + 2 + d] = a;
    if (d == 0) {
      r[g * (D + 2)] = M;
      r[g * (D + 2) + 1] = ls;
    }
  }
}

template <int D, int G>
__global__ void __launch_bounds__(256) k_dense_merge(StaticArgs A, int nsp) {
  constexpr int REC = G * (D + 2);
  const int u = blockIdx.x;
  const int b = u / A.Hkv, h = u % A.Hkv;
  const float* r = A.rec + static_cast<size_t>(u) * nsp * REC;
  for (int x = threadIdx.x; x < G * D; x += blockDim.x) {
    const int g = x / D, d = x % D;
    float M = -INFINITY;
    for (int s = 0; s < nsp; s++) M = fmaxf(M, r[s * REC + g * (D + 2)]);
    float a = 0.0f, ls = 0.0f;
    for (int s = 0; s < nsp; s++) {
      const float cw = exp_rel(r[s * REC + g * (D + 2)], M);
      a += r[s * REC + g * (D + 2) + 2 + d] * cw;
      ls += r[s * REC + g * (D + 2) + 1] * cw;
    }
    A.out[(static_cast<size_t>(b) * A.Hq + h * G + g) * D + d] = ls > 0.0f ? a / ls : 0.0f;
  }
}

typedef void (*SplitFn)(StaticArgs);
typedef void (*MergeFn)(StaticArgs, int);

template <typename T, int D>
bool pick_g(int G, SplitFn* s, MergeFn* m) {
  switch (G) {
    case 1: *s = k_dense_split<T, D, 1>; *m = k_dense_merge<D, 1>; return true;
    case 2: *s = k_dense_split<T, D, 2>; *m = k_dense_merge<D, 2>; return true;
    case 4: *s = k_dense_split<T, D, 4>; *m = k_dense_merge<D, 4>; return true;
    case 8: *s = k_dense_split<T, D, 8>; *m = k_dense_merge<D, 8>; return true;
    default: return false;
  }
}

bool pick(const vattn_config& c, int G, SplitFn* s, MergeFn* m) {
  if (c.dtype == VATTN_BF16)
    return c.head_dim == 128 ? pick_g<__nv_bfloat16, 128>(G, s, m) : pick_g<__nv_bfloat16, 64>(G, s, m);
  return c.head_dim == 128 ? pick_g<float, 128>(G, s, m) : pick_g<float, 64>(G, s, m);
}

// Per-context set-up: the address of this device's copy of the array, and
// its SM count, looked up by the first call made with a given CUDA context
// current on the device. The address belongs to the context that loaded the
// module, so the slot remembers that context's id and the look-up is redone
// when another context becomes current on the device (after
// cudaDeviceReset, or a context made by the driver API), instead of handing
// a kernel a stale address.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct DeviceSlot {
  bool ready;
  unsigned long long ctx_id;
  float* scratch;
  int num_sms;
};
std::mutex g_slots_mu;
DeviceSlot g_slots[kMaxDevices];

template <typename Fn>
Fn driver_entry(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Id of the context current on this thread (0 when none is current yet).
int current_ctx_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return VATTN_ECUDA;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS) return VATTN_ECUDA;
  *id = 0;
  if (c && get_id(c, id) != CUDA_SUCCESS) return VATTN_ECUDA;
  return VATTN_OK;
}

int device_slot(DeviceSlot* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VATTN_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return VATTN_EINVAL;
  unsigned long long id = 0;
  if (const int rc = current_ctx_id(&id)) return rc;
  std::lock_guard<std::mutex> lock(g_slots_mu);
  DeviceSlot& s = g_slots[dev];
  if (!s.ready || id == 0 || s.ctx_id != id) {
    // the look-up also makes the runtime's primary context current if none was
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dense_scratch) != cudaSuccess || p == nullptr) return VATTN_ECUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
      return VATTN_ECUDA;
    if (id == 0 && current_ctx_id(&id) != VATTN_OK) return VATTN_ECUDA;
    s.scratch = static_cast<float*>(p);
    s.num_sms = sms;
    s.ctx_id = id;
    s.ready = id != 0;
  }
  *out = s;
  return VATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int vattn_dense_decode_static(const vattn_config* cfg, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* page_table,
                                         const int32_t* seq_lens, int batch, int num_pages, float* out,
                                         void* stream) {
  // host checks first: a refused call touches neither the device nor the array
  if (!cfg || !q || !k_cache || !v_cache || !page_table || !seq_lens || !out) return VATTN_EINVAL;
  const vattn_config& c = *cfg;
  if (c.num_kv_heads < 1 || c.num_q_heads < 1 || c.num_q_heads % c.num_kv_heads) return VATTN_EINVAL;
  const int G = c.num_q_heads / c.num_kv_heads;
  if (!(G == 1 || G == 2 || G == 4 || G == 8)) return VATTN_EINVAL;
  if (!(c.head_dim == 64 || c.head_dim == 128)) return VATTN_EINVAL;
  if (!(c.dtype == VATTN_FP32 || c.dtype == VATTN_BF16)) return VATTN_EINVAL;
  if (c.page_size < 16 || c.page_size % 16) return VATTN_EINVAL;
  if (c.max_batch < 1 || c.max_ctx < 1 || c.max_ctx > (1 << 24)) return VATTN_EINVAL;
  if (batch < 0 || batch > c.max_batch || num_pages < 1) return VATTN_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return VATTN_EINVAL;
  if (c.kv_location != VATTN_KV_DEVICE && c.kv_location != VATTN_KV_HOST) return VATTN_EINVAL;
  const long long units = static_cast<long long>(batch) * c.num_kv_heads;
  const size_t rec_bytes = static_cast<size_t>(G) * (c.head_dim + 2) * sizeof(float);
  if (static_cast<size_t>(units) * rec_bytes > kStaticScratchBytes) return VATTN_ESCRATCH;
  if (batch == 0) return VATTN_OK;

  DeviceSlot slot;
  const int rc = device_slot(&slot);
  if (rc != VATTN_OK) return rc;
  if (c.kv_location == VATTN_KV_HOST) {  // page-locked host caches: their device addresses
    cudaPointerAttributes ak, av;
    if (cudaPointerGetAttributes(&ak, k_cache) != cudaSuccess || cudaPointerGetAttributes(&av, v_cache) != cudaSuccess) {
      cudaGetLastError();
      return VATTN_EINVAL;
    }
    if (ak.type != cudaMemoryTypeHost || av.type != cudaMemoryTypeHost || !ak.devicePointer || !av.devicePointer)
      return VATTN_EINVAL;
    k_cache = static_cast<const char*>(ak.devicePointer) +
              (static_cast<const char*>(k_cache) - static_cast<const char*>(ak.hostPointer ? ak.hostPointer : k_cache));
    v_cache = static_cast<const char*>(av.devicePointer) +
              (static_cast<const char*>(v_cache) - static_cast<const char*>(av.hostPointer ? av.hostPointer : v_cache));
  }
  SplitFn split;
  MergeFn merge;
  if (!pick(c, G, &split, &merge)) return VATTN_EINVAL;

  // splits per unit: about four CTAs per SM in all, at least 256 positions
  // each, and no more records than the array holds
  const long long want = (4LL * slot.num_sms + units - 1) / units;
  const long long by_len = (c.max_ctx + 255) / 256;
  const long long by_scratch = static_cast<long long>(kStaticScratchBytes / (static_cast<size_t>(units) * rec_bytes));
  const int nsp = static_cast<int>(std::max(1LL, std::min(want, std::min(by_len, by_scratch))));

  StaticArgs A;
  A.q = q;
  A.k = k_cache;
  A.v = v_cache;
  A.page_table = page_table;
  A.seq_lens = seq_lens;
  A.out = out;
  A.rec = slot.scratch;
  A.Hq = c.num_q_heads;
  A.Hkv = c.num_kv_heads;
  A.pps = (c.max_ctx + c.page_size - 1) / c.page_size;
  A.ps = c.page_size;
  A.max_ctx = c.max_ctx;
  A.num_pages = num_pages;
  A.scale = static_cast<float>(1.0 / sqrt(static_cast<double>(c.head_dim)));

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  split<<<dim3(nsp, static_cast<unsigned>(units)), kWarps * 32, 0, st>>>(A);
  merge<<<dim3(static_cast<unsigned>(units)), 256, 0, st>>>(A, nsp);
  return cudaGetLastError() == cudaSuccess ? VATTN_OK : VATTN_ECUDA;
}
