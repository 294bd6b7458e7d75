// Device-side building blocks of the decode step: element unpacking, the
// fixed-order fp32 dot, the order-preserving score key, Philox4x32-10, the
// fixed-order exp used by the budget statistics, and the shared parameter
// block every kernel receives.
//
// Arithmetic that decides an integer (ranking order, sample positions,
// budgets) is written with explicit round-to-nearest intrinsics so the
// compiler cannot contract or reorder it; see the comments at each function
// for the order it fixes.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vattn {

// bit of the device error word: a bounded wait in a kernel ran out
constexpr unsigned kDevTimeout = 4u;

constexpr int kHist1 = 2048;  // bins of digit 1 (key bits 31..21)
constexpr int kHist2 = 2048;  // bins of digit 2 (key bits 20..10)
constexpr int kHist3 = 1024;  // bins of digit 3 (key bits 9..0)
constexpr int kTopkSmem = 6144;    // top-k lists up to this length are staged in shared memory

// Per-unit (sequence b, KV head h) state written by the prep and budget kernels.
struct UnitInfo {
  int n;         // sequence length (0 when the sequence failed validation)
  int s1;        // end of the sinks: min(sinks, n)
  int wst;       // start of the window: max(n - window, s1)
  int k;         // top-k size, capped by the middle's length
  int p;         // pilot size
  int ntail;     // tail size: (wst - s1) - k
  int nI;        // |I_f| = s1 + k + (n - wst)
  int mode;      // 0: no tail; 1: tail taken whole without a pilot; 2: pilot + budget
  int bsz;       // final sample size b (ntail when the tail is taken whole)
  int exhausted; // 1 when the whole tail is taken with weight 1
  int nitems;    // entries gathered: nI + bsz
  int pad0;
  unsigned thr;  // top-k threshold key
  int need_eq;   // how many keys equal to thr (lowest positions first) are taken
  int pad1, pad2;
};

struct DevParams {
  // 2-D row maps of the K and V caches ([rows][D], one-row boxes) for the
  // row-gathering tensor copies; rows = num_pages * Hkv * page_size
  CUtensorMap tmk, tmv;
  // the same views in boxes of one row by 64 columns with the 128-byte
  // swizzle, for the tensor-core gathers (bf16 caches in device memory)
  CUtensorMap tmk_sw, tmv_sw;
  // shapes
  int Hq, Hkv, G, D;
  int pps;        // page-table entries per sequence
  int ps;         // page size (rows per page)
  unsigned long long ps_magic;  // ceil(2^64 / ps): j / ps = mulhi(j, ps_magic) for j < 2^24
  int max_ctx, batch, units, num_pages;
  int proxy, rank;
  // per-call parameters
  int sinks, window, topk_abs, topk_num, topk_den, pilot_min, pilot_num, pilot_den;
  float eps, scale;
  double z;
  unsigned long long seed;
  int dense;
  int guarantee;    // 1: the budget also bounds the numerator vector (output guarantee)
  int topp_num, topp_den;  // topp_den > 0: top-p selection with p = topp_num / topp_den
  int kv_host;      // 1: k and v point into mapped host memory (plain loads only)
  int batch_offset, head_offset;  // a shard's first sequence and KV head in the whole batch
  int CD, CS;       // grid sizes of the det (and dense) and sample gathers
  // inputs
  const void* q;
  const void* k;
  const void* v;
  const void* kt;
  const void* kp;
  const float* basis;
  const int* page_table;
  const int* seq_lens;
  // outputs
  float* out;
  int* sel;
  int* sel_count;
  int* budgets;
  int* head_need;
  // workspace
  UnitInfo* info;
  float* qbar;      // [units][D]: ranking query (group mean)
  float* qsel;      // [units][D]: SparQ query values at the chosen dims, or the Loki projected query
  int* dims;        // [units][D]: SparQ chosen dims, ascending
  unsigned* ordk;   // [units][max_ctx]: ranking-score keys over the middle
  unsigned* hist;   // [units][kHist1]: digit-1 histogram of the ranking keys
  float* pscore;    // [units][max_ctx][G]: true scores of I_f and the pilot
  int* num_need;    // [units][G]: numerator sizes n_v (output guarantee)
  long long* prefix;// [units + 1]: score-pass work prefix
  unsigned* gcnt;   // [0]: score-pass chunks handed out, [1]: units done by k_topp (zeroed by k_prep)
  long long* pre_det;   // [2 units + 1]: slice prefix of the det (or dense) gather
  long long* pre_samp;  // [2 units + 1]: slice prefix of the sample gather
  float* rec_det;   // [CD + 2 units][G][2 + D]: det (or dense) gather records
  float* rec_samp;  // [CS + 2 units][G][2 + D]: sample gather records
  unsigned* err;
};

// ---------------------------------------------------------------- elements
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPer16 = 4;
  __device__ static __forceinline__ void unpack(const uint4& r, float (&x)[4]) {
    x[0] = __uint_as_float(r.x);
    x[1] = __uint_as_float(r.y);
    x[2] = __uint_as_float(r.z);
    x[3] = __uint_as_float(r.w);
  }
  __device__ static __forceinline__ float load(const void* base, size_t i) {
    return static_cast<const float*>(base)[i];
  }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kPer16 = 8;
  // word w holds element 2w in its low half and 2w+1 in its high half
  __device__ static __forceinline__ void unpack(const uint4& r, float (&x)[8]) {
    x[0] = __uint_as_float(r.x << 16);
    x[1] = __uint_as_float(r.x & 0xFFFF0000u);
    x[2] = __uint_as_float(r.y << 16);
    x[3] = __uint_as_float(r.y & 0xFFFF0000u);
    x[4] = __uint_as_float(r.z << 16);
    x[5] = __uint_as_float(r.z & 0xFFFF0000u);
    x[6] = __uint_as_float(r.w << 16);
    x[7] = __uint_as_float(r.w & 0xFFFF0000u);
  }
  __device__ static __forceinline__ float load(const void* base, size_t i) {
    return __uint_as_float(static_cast<unsigned>(static_cast<const unsigned short*>(base)[i]) << 16);
  }
};

// Streaming 16-byte load (cache-streaming: likely accessed once).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  return __ldcs(static_cast<const uint4*>(p));
}

// Read-only 16-byte load for gathered rows.
__device__ __forceinline__ uint4 ld_gather(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------- fixed-order dot
// One 16-byte chunk of the dot: a fused multiply-add chain from 0 over the
// chunk's elements in ascending order.
template <typename T>
__device__ __forceinline__ float chunk_dot(const float* q, const uint4& raw) {
  constexpr int E = Elem<T>::kPer16;
  float x[E];
  Elem<T>::unpack(raw, x);
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < E; i++) acc = __fmaf_rn(q[i], x[i], acc);
  return acc;
}

__host__ __device__ constexpr int ilog2c(int x) { return x <= 1 ? 0 : 1 + ilog2c(x / 2); }

// Chunk sums of U rows live in the L lanes of an aligned lane group (lane li
// holds chunk li of every row). Each row's dot is the halving-stride tree over
// chunks: chunk l += chunk l + L/2, then l += l + L/4, ..., l += l + 1. At the
// first log2(U) stages each lane keeps half of its rows and receives its
// partner's partials for them, so U rows cost (U - 1) + log2(L/U) shuffles
// instead of U*log2(L); every stage still adds the partials of lanes x and
// x^o for a row (fp addition is commutative), so each row's sum is exactly
// that tree. Afterwards the lanes [r*(L/U), (r+1)*(L/U)) of the group hold
// row r (U <= L).
template <int L, int U>
__device__ __forceinline__ float reduce_rows(float (&a)[U], int li) {
  constexpr int LOGL = ilog2c(L);
  constexpr int LOGU = ilog2c(U);
#pragma unroll
  for (int s = 0; s < LOGL; s++) {
    const int o = L >> (s + 1);
    if (s < LOGU) {
      const int half = U >> (s + 1);
      const bool up = (li & o) != 0;
#pragma unroll
      for (int i = 0; i < half; i++) {
        float send = up ? a[i] : a[i + half];
        float keep = up ? a[i + half] : a[i];
        a[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, o));
      }
    } else {
      a[0] = __fadd_rn(a[0], __shfl_xor_sync(0xffffffffu, a[0], o));
    }
  }
  return a[0];
}

template <int L, int U>
__device__ __forceinline__ int reduce_rows_row(int li) {
  constexpr int LOGU = ilog2c(U);
  int r = 0;
#pragma unroll
  for (int s = 0; s < LOGU; s++) {
    const int o = L >> (s + 1);
    if (li & o) r += U >> (s + 1);
  }
  return r;
}

// ---------------------------------------------------------------- keys
// Order-preserving map of an fp32 score onto uint32; -0 maps like +0.
__device__ __forceinline__ unsigned ord_key(float f) {
  if (f == 0.0f) f = 0.0f;
  unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- Philox4x32-10
// Salmon, Moraes, Dror, Shaw (SC'11). Draw t of unit (b, h) is word t%4 of the
// block with counter (t/4, b, h, 0) under key (seed low, seed high).
__device__ __forceinline__ uint4 draw_block(unsigned long long seed, unsigned b, unsigned h, unsigned blk) {
  unsigned c0 = blk, c1 = b, c2 = h, c3 = 0u;
  unsigned k0 = static_cast<unsigned>(seed), k1 = static_cast<unsigned>(seed >> 32);
#pragma unroll
  for (int round = 0; round < 10; round++) {
    if (round > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const unsigned lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
    const unsigned lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
    const unsigned n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}
__device__ __forceinline__ unsigned draw_word(unsigned long long seed, unsigned b, unsigned h,
                                              unsigned t) {
  const uint4 q = draw_block(seed, b, h, t >> 2);
  const unsigned w = t & 3u;
  return w == 0 ? q.x : (w == 1 ? q.y : (w == 2 ? q.z : q.w));
}

// Lemire multiply-shift: a 32-bit uniform word onto [0, n).
__device__ __forceinline__ int lemire(unsigned u, int n) {
  return static_cast<int>((static_cast<unsigned long long>(u) * static_cast<unsigned>(n)) >> 32);
}

// ---------------------------------------------------------------- fixed-order exp
// e^x for x <= 0 in fp32 (Cody-Waite): n = rint(x*log2 e); r = (x - n*C1) - n*C2
// with ln 2 = C1 + C2, C1 = 0.693359375 (9 significant bits, so n*C1 is exact);
// e^r by its degree-7 Taylor polynomial in Horner form with fused steps;
// result p * 2^n. Below -87 the result leaves the normal range and 0 is
// returned. Used only where the value feeds the integer budget statistics.
__device__ __forceinline__ float vexp(float x) {
  if (!(x >= -87.0f)) return 0.0f;
  const float n = rintf(__fmul_rn(x, 1.44269504088896341f));
  float r = __fmaf_rn(-n, 0.693359375f, x);
  r = __fmaf_rn(-n, -2.12194440054690583e-4f, r);
  float p = 1.98412698412698413e-4f;           // 1/7!
  p = __fmaf_rn(p, r, 1.38888888888888889e-3f); // 1/6!
  p = __fmaf_rn(p, r, 8.33333333333333333e-3f); // 1/5!
  p = __fmaf_rn(p, r, 4.16666666666666667e-2f); // 1/4!
  p = __fmaf_rn(p, r, 1.66666666666666667e-1f); // 1/3!
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const float scale = __int_as_float((static_cast<int>(n) + 127) << 23);
  return __fmul_rn(p, scale);
}

// ---------------------------------------------------------------- block helpers
// Inclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ unsigned block_inclusive_scan(unsigned v, unsigned* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    unsigned w = lane < nw ? s_warp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < nw) s_warp[lane] = w;
  }
  __syncthreads();
  const unsigned base = warp > 0 ? s_warp[warp - 1] : 0u;
  __syncthreads();
  return v + base;
}

// Radix-select step over a shared-memory histogram, for any block of BT
// threads: find the bin holding the krem-th largest key (counting from the
// top bin) and the rank left inside that bin; each thread scans NB / BT
// consecutive bins downwards.
template <int NB, int BT>
__device__ __forceinline__ void find_digit_bt(const unsigned* hist, int krem, int* s_digit, int* s_krem,
                                              unsigned* s_warp) {
  constexpr int PER = NB / BT;
  static_assert(PER >= 1 && NB % BT == 0, "bins per thread");
  const int lo = NB - (threadIdx.x + 1) * PER;
  unsigned v[PER];
  unsigned sum = 0;
#pragma unroll
  for (int i = 0; i < PER; i++) {
    v[i] = hist[lo + i];
    sum += v[i];
  }
  const unsigned incl = block_inclusive_scan(sum, s_warp);
  const unsigned excl = incl - sum;
  if (excl < static_cast<unsigned>(krem) && static_cast<unsigned>(krem) <= incl) {
    unsigned c = excl;
    bool done = false;
#pragma unroll
    for (int i = PER - 1; i >= 0; i--) {
      if (!done && c + v[i] >= static_cast<unsigned>(krem)) {
        *s_digit = lo + i;
        *s_krem = krem - static_cast<int>(c);
        done = true;
      }
      c += v[i];
    }
  }
  __syncthreads();
}

}  // namespace vattn
