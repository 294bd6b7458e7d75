// Kernels of one verified-sparse-attention decode step, in launch order:
//
//   k_prep        per unit: validate, regions, ranking query, proxy query,
//                 zero the digit-1 histogram, write sinks/window indices; one
//                 extra CTA writes the score-pass work prefix and the det
//                 gather's slice prefix
//   k_score_tma   exact or Loki ranking scores of a contiguous cache, streamed
//   k_score_rows  through bulk copies (k_score_rows: paged caches, or caches
//   k_score_sparq in host memory; k_score_sparq: the SparQ proxy from the
//                 dim-major K copy); writes the order keys and the histogram
//                 of their first radix digit
//   k_topp        (top-p only) each unit's top-k size from its scores' mass
//   k_topk        top-k select and pilot draws, one CTA per unit, the keys
//                 streamed from L2
//   k_gather<det>    gather + softmax-accumulate of I_f and the pilot draws
//                    (true scores of every query head kept)
//   k_numstats    (output guarantee only) numerator statistics of the pilot
//   k_budget      per-head CLT budgets from the pilot statistics
//   k_draws       the rest of the sample's positions; the sample slice prefix
//   k_gather<sample> the remaining draws (or the whole tail)
//   k_combine<sample> merge the records, reweight the sample by N_tail / b,
//                    write out (k_gather<dense> + k_combine<dense>: dense decode)
//
// A unit is one (sequence b, KV head h); u = b * Hkv + h. The method follows
// "vAttention: A New Approach to Sparse Attention with Guaranteed Accuracy",
// section "How vAttention Works" and the paragraph after it.
#pragma once

#include <cooperative_groups.h>

#include "vattn_device.cuh"

namespace vattn {

constexpr int kProxyExact = 0, kProxySparq = 1, kProxyLoki = 2;

// Page-table slot of position j (exact for 0 <= j < 2^24, page size >= 2).
__device__ __forceinline__ int page_slot(const DevParams& P, int j) {
  return static_cast<int>(__umul64hi(static_cast<unsigned long long>(j), P.ps_magic));
}

// Element offset of row j of unit (b, h) in a [pages][Hkv][page_size][W] cache.
__device__ __forceinline__ size_t row_off(const DevParams& P, int b, int h, int j, int W) {
  const int slot = page_slot(P, j);
  const size_t page = static_cast<size_t>(P.page_table[static_cast<size_t>(b) * P.pps + slot]);
  const int row = j - slot * P.ps;
  return ((page * P.Hkv + h) * P.ps + row) * static_cast<size_t>(W);
}

// Regions of a sequence of length n (sinks [0,s1), middle [s1,wst), window [wst,n)).
struct Regions {
  int s1, wst, k, p;
};
__device__ __forceinline__ Regions regions(const DevParams& P, int n) {
  Regions r;
  r.s1 = min(P.sinks, n);
  r.wst = max(n - P.window, r.s1);
  const int mlen = r.wst - r.s1;
  // with top-p the size is found after the score pass (k_topp); 0 until then
  const long long kb = P.topp_den ? 0LL
                       : P.topk_den ? (static_cast<long long>(n) * P.topk_num) / P.topk_den
                                    : static_cast<long long>(P.topk_abs);
  r.k = static_cast<int>(min(kb, static_cast<long long>(mlen)));
  long long pb = P.pilot_min;
  if (P.pilot_den) {
    const long long c = (static_cast<long long>(n) * P.pilot_num + P.pilot_den - 1) / P.pilot_den;
    pb = max(pb, c);
  }
  r.p = static_cast<int>(pb);
  return r;
}

// Score-pass work items of a unit: rows of the middle, or, for SparQ, aligned
// groups of V positions covering it.
__device__ __forceinline__ long long score_work(const DevParams& P, int n, int V) {
  const Regions r = regions(P, n);
  if (r.wst <= r.s1) return 0;
  if (P.proxy != kProxySparq) return r.wst - r.s1;
  return (r.wst + V - 1) / V - r.s1 / V;
}

// ---------------------------------------------------------------- launch chaining
// Every kernel is launched with programmatic dependent launch: it may start
// while its predecessor finishes, and waits here before touching anything the
// predecessor wrote (no-op when launched without the attribute).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the successor launch once every CTA of this grid has passed this point.
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ============================================================ k_prep
constexpr int kPrepLens = 1024;  // sequence lengths the prefix CTA keeps in shared memory

template <typename T, int D, int G>
__global__ void __launch_bounds__(128) k_prep(DevParams P) {
  __shared__ float s_q[D];
  __shared__ float s_abs[D];
  __shared__ unsigned s_warp[32];
  __shared__ unsigned s_tot;
  const int tid = threadIdx.x;
  const int u = blockIdx.x;
  grid_dependency_wait();  // the previous call's kernels still read this workspace

  if (u == P.units) {
    // the validated lengths once into shared memory (the scans below then run
    // without a global load per round)
    __shared__ int s_len[kPrepLens];
    auto seq_len = [&](int bq) -> int {
      int n = bq < kPrepLens ? s_len[bq] : P.seq_lens[bq];
      if (bq >= kPrepLens && (n < 0 || n > P.max_ctx)) n = 0;
      return n;
    };
    for (int i = tid; i < min(P.batch, kPrepLens); i += blockDim.x) {
      const int n = P.seq_lens[i];
      s_len[i] = (n < 0 || n > P.max_ctx) ? 0 : n;
    }
    __syncthreads();
    // work prefix over units for the persistent score pass
    constexpr int V = Elem<T>::kPer16;
    long long carry = 0;
    for (int base = 0; base < P.units; base += blockDim.x) {
      const int uu = base + tid;
      long long w = 0;
      if (uu < P.units) w = score_work(P, seq_len(uu / P.Hkv), V);
      // work per unit <= max_ctx <= 2^24, so a 128-unit chunk sum fits in 32 bits
      const unsigned incl = block_inclusive_scan(static_cast<unsigned>(w), s_warp);
      if (uu < P.units) P.prefix[uu] = carry + (incl - static_cast<unsigned>(w));
      if (tid == blockDim.x - 1) s_tot = incl;
      __syncthreads();
      carry += s_tot;
      __syncthreads();
    }
    if (tid == 0) P.prefix[P.units] = carry;
    // slice prefix of the det (or dense) gather, from the length-checked n; a
    // sequence whose pages fail validation keeps its items here and is
    // skipped by the gather, which reads the validated unit state
    carry = 0;
    const int ns = 2 * P.units;
    for (int base = 0; base < ns; base += blockDim.x) {
      const int sidx = base + tid;
      unsigned cnt = 0;
      if (sidx < ns) {
        const int n = seq_len((sidx >> 1) / P.Hkv);
        if (P.dense) {
          cnt = (sidx & 1) ? 0u : static_cast<unsigned>(n);
        } else {
          const Regions r = regions(P, n);
          const int ntail = (r.wst - r.s1) - r.k;
          const int nI = r.s1 + r.k + (n - r.wst);
          const int mode = ntail == 0 ? 0 : (ntail <= r.p ? 1 : 2);
          const int n_extra = mode == 2 ? r.p : (mode == 1 ? ntail : 0);
          const int n_det = mode == 2 ? nI : nI + n_extra;
          cnt = static_cast<unsigned>((sidx & 1) ? nI + n_extra - n_det : n_det);
        }
      }
      const unsigned incl = block_inclusive_scan(cnt, s_warp);
      if (sidx < ns) P.pre_det[sidx] = carry + (incl - cnt);
      if (tid == blockDim.x - 1) s_tot = incl;
      __syncthreads();
      carry += s_tot;
      __syncthreads();
    }
    if (tid == 0) {
      P.pre_det[ns] = carry;
      P.gcnt[0] = 0u;
      P.gcnt[1] = 0u;
    }
    return;
  }

  const int b = u / P.Hkv, h = u % P.Hkv;
  int n = P.seq_lens[b];
  const bool bad_len = n < 0 || n > P.max_ctx;
  if (bad_len) n = 0;
  const int npages = (n + P.ps - 1) / P.ps;
  int bad = 0;
  for (int i0 = tid; i0 < npages; i0 += 8 * blockDim.x) {  // eight independent loads in flight
    int pid[8];
#pragma unroll
    for (int j = 0; j < 8; j++) {
      const int i = i0 + j * blockDim.x;
      pid[j] = i < npages ? P.page_table[static_cast<size_t>(b) * P.pps + i] : 0;
    }
#pragma unroll
    for (int j = 0; j < 8; j++)
      if (pid[j] < 0 || pid[j] >= P.num_pages) bad = 1;
  }
  bad = __syncthreads_or(bad);
  if (tid == 0 && h == 0) {
    if (bad_len) atomicOr(P.err, 1u);
    if (bad) atomicOr(P.err, 2u);
  }
  if (bad) n = 0;

  const Regions r = regions(P, n);
  const int mlen = r.wst - r.s1;
  const int ntail = mlen - r.k;
  const int nI = r.s1 + r.k + (n - r.wst);
  if (tid == 0) {
    UnitInfo inf;
    inf.n = n;
    inf.s1 = r.s1;
    inf.wst = r.wst;
    inf.k = r.k;
    inf.p = r.p;
    inf.ntail = ntail;
    inf.nI = nI;
    inf.mode = ntail == 0 ? 0 : (ntail <= r.p ? 1 : 2);
    inf.bsz = 0;
    inf.exhausted = 0;
    inf.nitems = nI;
    inf.pad0 = 0;
    inf.thr = 0xFFFFFFFFu;
    inf.need_eq = 0;
    inf.pad1 = inf.pad2 = 0;
    P.info[u] = inf;
  }

  // Ranking query: pairwise tree over adjacent heads of the group, then x 1/G.
  if (tid < D) {
    float v[G];
#pragma unroll
    for (int g = 0; g < G; g++)
      v[g] = Elem<T>::load(P.q, (static_cast<size_t>(b) * P.Hq + h * G + g) * D + tid);
#pragma unroll
    for (int stride = 1; stride < G; stride *= 2)
#pragma unroll
      for (int g = 0; g + stride < G; g += 2 * stride) v[g] = __fadd_rn(v[g], v[g + stride]);
    const float qb = __fmul_rn(v[0], 1.0f / static_cast<float>(G));
    s_q[tid] = qb;
    s_abs[tid] = fabsf(qb);
    P.qbar[static_cast<size_t>(u) * D + tid] = qb;
  }
  __syncthreads();

  if (P.proxy == kProxySparq) {
    // the r components of largest magnitude (ties to the lower dim), ascending
    int sel = 0;
    if (tid < D) {
      const float a = s_abs[tid];
      int rank = 0;
      for (int j = 0; j < D; j++) {
        const float bj = s_abs[j];
        rank += (bj > a) || (bj == a && j < tid);
      }
      sel = rank < P.rank;
    }
    const unsigned incl = block_inclusive_scan(static_cast<unsigned>(sel), s_warp);
    if (sel) {
      const int pos = static_cast<int>(incl) - 1;
      P.dims[static_cast<size_t>(u) * D + pos] = tid;
      P.qsel[static_cast<size_t>(u) * D + pos] = s_q[tid];
    }
  } else if (P.proxy == kProxyLoki) {
    // projected ranking query: one fused chain over d per component
    // the head's basis (d x 32 fp32) into shared memory by every thread at
    // once, then one chain per component over it in order
    __shared__ float s_basis[D * 32];
    const float* basis = P.basis + static_cast<size_t>(h) * D * P.rank;
    const int nb = D * P.rank;  // rank is 32
    for (int i0 = tid; i0 < nb; i0 += 8 * blockDim.x) {
      float bv[8];
#pragma unroll
      for (int j = 0; j < 8; j++) bv[j] = i0 + j * blockDim.x < nb ? basis[i0 + j * blockDim.x] : 0.0f;
#pragma unroll
      for (int j = 0; j < 8; j++)
        if (i0 + j * blockDim.x < nb) s_basis[i0 + j * blockDim.x] = bv[j];
    }
    __syncthreads();
    if (tid < P.rank) {
      float acc = 0.0f;
      for (int i = 0; i < D; i++) acc = __fmaf_rn(s_q[i], s_basis[i * P.rank + tid], acc);
      P.qsel[static_cast<size_t>(u) * D + tid] = acc;
    }
  }

  unsigned* hist = P.hist + static_cast<size_t>(u) * kHist1;
  for (int i = tid; i < kHist1; i += blockDim.x) hist[i] = 0u;
  int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx;
  for (int i = tid; i < r.s1; i += blockDim.x) sel[i] = i;
  if (P.topp_den == 0)  // with top-p, k_topp writes the window once k is known
    for (int i = tid; i < n - r.wst; i += blockDim.x) sel[r.s1 + r.k + i] = r.wst + i;
}

// ============================================================ score pass helpers
// Share of the score pass's rows split statically over the CTAs, and the
// bytes of rows per dynamically handed-out chunk of the rest (CTAs that
// stream faster take more of it; the counter is zeroed by k_prep). The bulk-
// copy pass over contiguous caches streams more evenly and takes the larger
// static share (measured best of 0.6-1.0 for each pass).
constexpr double kScoreStatic = 0.8;
constexpr double kScoreStaticTma = 0.9;
constexpr long long kScoreChunkBytes = 262144;

// The whole block searches the prefix in one round of loads: the unit
// whose non-empty range [prefix[u], prefix[u+1]) holds x (0 if none).
__device__ __forceinline__ int find_unit_block(const long long* prefix, int units, long long x, int* s_u) {
  if (threadIdx.x == 0) *s_u = 0;
  __syncthreads();
  for (int v = threadIdx.x; v < units; v += blockDim.x)
    if (prefix[v] <= x && x < prefix[v + 1]) *s_u = v;
  __syncthreads();
  return *s_u;
}

__device__ __forceinline__ void flush_hist(unsigned* s_hist, unsigned* g_hist) {
  __syncthreads();
  for (int i = threadIdx.x; i < kHist1; i += blockDim.x) {
    const unsigned c = s_hist[i];
    if (c) atomicAdd(g_hist + i, c);
    s_hist[i] = 0u;
  }
  __syncthreads();
}

// ============================================================ k_score_rows
// Exact mode (W = D, query = group mean, rows of K) and Loki mode (W = rank,
// query = projected query, rows of the projected-key cache). Each row of W
// elements is split over L lanes (16 bytes each); a warp covers RPW rows per
// load instruction and every lane group keeps U rows in flight.
template <typename T, int W>
__global__ void __launch_bounds__(256) k_score_rows(DevParams P) {
  constexpr int E = Elem<T>::kPer16;
  constexpr int L = W / E;
  constexpr int RPW = 32 / L;
  constexpr int U = L < 8 ? L : 8;
  constexpr int ROWS_WARP = RPW * U;
  static_assert(L >= 2 && L <= 32 && (L & (L - 1)) == 0, "row must be 2..32 chunks");
  __shared__ unsigned s_hist[kHist1];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int grp = lane / L, li = lane % L;
  grid_dependency_wait();
  const bool loki = P.proxy == kProxyLoki;
  const void* cache = loki ? P.kp : P.k;
  const float* qsrc = loki ? P.qsel : P.qbar;

  for (int i = threadIdx.x; i < kHist1; i += blockDim.x) s_hist[i] = 0u;
  __syncthreads();

  const long long total = P.prefix[P.units];
  // static share in equal ranges, the rest in chunks from an atomic counter
  const long long tstat = static_cast<long long>(static_cast<double>(total) * kScoreStatic);
  constexpr long long kChunk = kScoreChunkBytes / (W * static_cast<long long>(sizeof(T)));
  const long long nchunk = (total - tstat + kChunk - 1) / kChunk;
  __shared__ int s_u;
  __shared__ long long s_chunk;
  long long beg = tstat * blockIdx.x / gridDim.x;
  long long end = tstat * (blockIdx.x + 1) / gridDim.x;
  for (;;) {
  if (beg < end) {
  int u = find_unit_block(P.prefix, P.units, beg, &s_u);
  long long cur = beg;
  while (cur < end) {
    while (P.prefix[u + 1] <= cur) u++;
    const long long uend = min(end, P.prefix[u + 1]);
    const UnitInfo inf = P.info[u];
    if (inf.n > 0) {
      const int b = u / P.Hkv, h = u % P.Hkv;
      const int j0 = inf.s1 + static_cast<int>(cur - P.prefix[u]);
      const int j1 = inf.s1 + static_cast<int>(uend - P.prefix[u]);
      float q[E];
#pragma unroll
      for (int e = 0; e < E; e++) q[e] = qsrc[static_cast<size_t>(u) * P.D + li * E + e];
      const T* base = static_cast<const T*>(cache);
      unsigned* ordk = P.ordk + static_cast<size_t>(u) * P.max_ctx;
      for (int jb = j0 + warp * ROWS_WARP; jb < j1; jb += nwarps * ROWS_WARP) {
        uint4 raw[U];
#pragma unroll
        for (int k = 0; k < U; k++) {
          const int j = jb + k * RPW + grp;
          if (j < j1)
            raw[k] = ld_stream(base + row_off(P, b, h, j, W) + li * E);
          else
            raw[k] = make_uint4(0u, 0u, 0u, 0u);
        }
        float a[U];
#pragma unroll
        for (int k = 0; k < U; k++) a[k] = chunk_dot<T>(q, raw[k]);
        const float s = reduce_rows<L, U>(a, li);
        const int r = reduce_rows_row<L, U>(li);
        const int j = jb + r * RPW + grp;
        if ((li % (L / U)) == 0 && j < j1) {
          const unsigned o = ord_key(s);
          ordk[j] = o;
          atomicAdd(&s_hist[o >> 21], 1u);
        }
      }
      flush_hist(s_hist, P.hist + static_cast<size_t>(u) * kHist1);
    }
    cur = uend;
  }
  }
  __syncthreads();
  if (threadIdx.x == 0) s_chunk = static_cast<long long>(atomicAdd(P.gcnt, 1u));
  __syncthreads();
  const long long c = s_chunk;
  if (c >= nchunk) break;
  beg = tstat + c * kChunk;
  end = min(total, beg + kChunk);
  }
}

// ============================================================ k_score_sparq
// SparQ proxy: r_j = sum over the chosen dims i (ascending) of qbar_i * K[j][i],
// one fused chain per position, read from the dim-major copy. Each thread
// scores V consecutive positions (one 16-byte vector per dim).
template <typename T, int D>
__global__ void __launch_bounds__(256) k_score_sparq(DevParams P) {
  constexpr int V = Elem<T>::kPer16;
  __shared__ unsigned s_hist[kHist1];
  __shared__ float s_qv[D];
  __shared__ int s_dim[D];

  grid_dependency_wait();
  for (int i = threadIdx.x; i < kHist1; i += blockDim.x) s_hist[i] = 0u;
  __syncthreads();
  const long long total = P.prefix[P.units];
  const long long beg = total * blockIdx.x / gridDim.x;
  const long long end = total * (blockIdx.x + 1) / gridDim.x;
  if (beg >= end) return;
  const int r = P.rank;
  __shared__ int s_u;
  int u = find_unit_block(P.prefix, P.units, beg, &s_u);
  long long cur = beg;
  while (cur < end) {
    while (P.prefix[u + 1] <= cur) u++;
    const long long uend = min(end, P.prefix[u + 1]);
    const UnitInfo inf = P.info[u];
    if (inf.n > 0) {
      const int b = u / P.Hkv, h = u % P.Hkv;
      __syncthreads();
      for (int i = threadIdx.x; i < r; i += blockDim.x) {
        s_qv[i] = P.qsel[static_cast<size_t>(u) * D + i];
        s_dim[i] = P.dims[static_cast<size_t>(u) * D + i];
      }
      __syncthreads();
      const long long g0 = inf.s1 / V;
      const long long gb = g0 + (cur - P.prefix[u]), ge = g0 + (uend - P.prefix[u]);
      const T* kt = static_cast<const T*>(P.kt);
      unsigned* ordk = P.ordk + static_cast<size_t>(u) * P.max_ctx;
      for (long long gi = gb + threadIdx.x; gi < ge; gi += blockDim.x) {
        const int j0 = static_cast<int>(gi) * V;
        const int slot = page_slot(P, j0);
        const size_t page = static_cast<size_t>(P.page_table[static_cast<size_t>(b) * P.pps + slot]);
        const size_t ps = static_cast<size_t>(P.ps);
        const size_t rowbase = (page * P.Hkv + h) * D * ps;
        const int off = j0 - slot * P.ps;
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; v++) acc[v] = 0.0f;
        int t = 0;
        constexpr int NB = 16;  // dims loaded together (16-byte vectors in flight per thread)
        for (; t + NB <= r; t += NB) {
          uint4 raw[NB];
#pragma unroll
          for (int c = 0; c < NB; c++)
            raw[c] = ld_stream(kt + rowbase + static_cast<size_t>(s_dim[t + c]) * ps + off);
#pragma unroll
          for (int c = 0; c < NB; c++) {
            float x[V];
            Elem<T>::unpack(raw[c], x);
            const float qv = s_qv[t + c];
#pragma unroll
            for (int v = 0; v < V; v++) acc[v] = __fmaf_rn(qv, x[v], acc[v]);
          }
        }
        for (; t < r; t++) {
          const uint4 raw = ld_stream(kt + rowbase + static_cast<size_t>(s_dim[t]) * ps + off);
          float x[V];
          Elem<T>::unpack(raw, x);
          const float qv = s_qv[t];
#pragma unroll
          for (int v = 0; v < V; v++) acc[v] = __fmaf_rn(qv, x[v], acc[v]);
        }
#pragma unroll
        for (int v = 0; v < V; v++) {
          const int j = j0 + v;
          if (j >= inf.s1 && j < inf.wst) {
            const unsigned o = ord_key(acc[v]);
            ordk[j] = o;
            atomicAdd(&s_hist[o >> 21], 1u);
          }
        }
      }
      flush_hist(s_hist, P.hist + static_cast<size_t>(u) * kHist1);
    }
    cur = uend;
  }
}

// ============================================================ tail positions
// Position of the rho-th tail element (0-based, ascending) of M minus top-k:
// s1 + rho + c, with c the number of top-k entries t_i with t_i - s1 - i <= rho.
__device__ __forceinline__ int tail_position(const int* topk, int k, int s1, int rho) {
  int lo = 0, hi = k;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (topk[mid] - s1 - mid <= rho) lo = mid + 1; else hi = mid;  // topk: shared or global memory
  }
  return s1 + rho + lo;
}

// ============================================================ gathers
// One kernel template, three modes, each a persistent grid over a flattened
// list of items. Items are grouped in slices, two per unit (u, part): part 0
// carries weight 1, part 1 is sample. pre[s] is the prefix of item counts
// over slices s = 2u + part; CTA c of C owns items [c*T/C, (c+1)*T/C) of the
// T in total and writes one record per slice it touches, at index c + s
// (unique: along the flattened order both c and s only grow, and one of them
// grows at every segment boundary).
//   det:    part 0 = I_f (or all of I_f and the tail when the tail is no
//           larger than the pilot); part 1 = the p pilot draws. True scores
//           of every query head go to pscore for the budget.
//   sample: part 0 = the whole tail when the budget covers it; part 1 = the
//           draws t in [p, b).
//   dense:  part 0 = every position.
constexpr int kModeDet = 0, kModeSample = 1, kModeDense = 2;

// Each warp streams its blocks of R rows through a private ring of NS
// shared-memory stages: one lane per row issues two bulk copies (the K row
// and the V row) that complete on the stage's mbarrier, NS - 1 blocks ahead
// of the block being computed, so the bytes in flight live in shared memory
// rather than registers. In a block, a row is NC = D / E lanes wide (one
// 16-byte chunk each) and a warp step covers RPW = 32 / NC rows; UNR steps
// make a block. Every lane computes its chunk's partial dot product for all
// UNR rows and G heads (V = UNR * G values); one transposed reduction over
// the NC lanes of a row then leaves each lane owning whole dot products (the
// chunk sums are added pairwise at halving strides, the same tree as the
// scoring order). The block's softmax weights go through shared memory to the
// lanes that accumulate V.
template <typename T, int D, int G>
struct GatherShape {
  static constexpr int E = Elem<T>::kPer16;        // elements per 16-byte chunk
  static constexpr int NC = D / E;                 // chunks (lanes) per row
  static constexpr int LOGNC = ilog2c(NC);
  static constexpr int RPW = 32 / NC;              // rows per warp step
  static constexpr int UNR = G >= 8 ? 4 : 8;       // steps per block
  static constexpr int R = RPW * UNR;              // rows per block
  static constexpr int ROWB = D * static_cast<int>(sizeof(T));
  static constexpr int BLKB = 2 * R * ROWB;        // K rows, then V rows (4 or 8 KB)
  static constexpr int NW = 8;                     // warps per CTA
  static constexpr int NS = (192 * 1024) / (NW * BLKB);  // stages filling a 192 KB ring
  static constexpr int V = UNR * G;                // partial dot products per lane
  static constexpr int LOGV = ilog2c(V);
  static constexpr int NVF = LOGV >= LOGNC ? (V >> LOGNC) : 1;             // owned per lane
  static constexpr int REP = LOGV >= LOGNC ? 1 : (1 << (LOGNC - LOGV));    // lanes per score
  static constexpr int REC = G * (2 + D);          // floats per record: (m, l, acc[D]) per head
  static constexpr int WSP = 3 * R * G + 2 * G;    // per-warp floats: scores, weight pairs, (m, cf)
  static constexpr size_t RING = static_cast<size_t>(NW) * NS * BLKB;
  static constexpr size_t OFF_SP = RING;
  static constexpr size_t OFF_L = OFF_SP + static_cast<size_t>(NW) * WSP * 4;
  static constexpr size_t OFF_BAR = OFF_L + static_cast<size_t>(NW) * 32 * NVF * 4;
  static constexpr size_t SMEM = OFF_BAR + static_cast<size_t>(NW) * NS * 8;
  static_assert(OFF_BAR % 8 == 0, "mbarriers need 8-byte alignment");
  static_assert(SMEM <= 227 * 1024, "gather shared memory");
};

// exp(x - m) with m a running maximum (0 while m is still -inf).
__device__ __forceinline__ float exp_rel(float x, float m) {
  return m == -INFINITY ? 0.0f : __expf(x - m);
}

__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Makes barrier initialisation visible to the async proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Plain arrival (no transaction bytes): completes a phase whose stage was
// filled by ordinary stores.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// Bounded wait for the completion of the barrier phase with parity `parity`;
// false when `tries` tries ran out (each try may itself suspend for a while,
// so the default limit ends a wait that can never complete in about a second).
// A warp whose wait failed issues no further copies into its ring and first
// waits once more, with the same limit, for every block it still has in
// flight (drain_ring), so that no copy lands in shared memory after it has
// moved on; a wait can only fail after a copy that never completes, which the
// row bounds of every copy rule out in normal operation.
constexpr int kWaitTries = 1 << 20;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, int tries = kWaitTries) {
  const unsigned a = smem_u32(bar);
  for (int it = 0; it < tries; it++) {
    unsigned done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
// Orders this thread's earlier generic shared-memory accesses before later
// async-proxy writes (a bulk copy into a stage that was just read).
// Bounded waits for blocks [t, nis) of a slice (ring stage and phase from
// the running block count issued + t), after the wait on block t failed.
__device__ __noinline__ void drain_ring(uint64_t* bars, int NS, unsigned issued, int t, int nis) {
  for (int t2 = t; t2 < nis; t2++) {
    const unsigned g = issued + static_cast<unsigned>(t2);
    mbar_wait(&bars[g % NS], (g / NS) & 1u);
  }
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  const size_t g = __cvta_generic_to_global(src);
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(g), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Tensor copy of four rows (row indices y0..y3, all columns of a one-row
// box) of the 2-D row map `map` into consecutive rows at dst, completing on
// `bar`.
__device__ __forceinline__ void gather4_g2s(void* dst, const CUtensorMap* map, int y0, int y1, int y2, int y3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(0), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}

// Transposed reduction of NV values per lane over the lanes that differ in
// bits O, O/2, ..., 1 of the lane index: while a lane holds more than one
// value it keeps one half (the upper half when its bit O is set) and adds the
// partner's copy of that half; once it holds one value, the remaining levels
// are plain butterflies. Every sum pairs the same two subtrees as the halving
// tree over chunks.
template <int NV, int O>
struct TReduce {
  __device__ static __forceinline__ void run(float* x, int lane) {
    if constexpr (O >= 1) {
      if constexpr (NV > 1) {
        const bool hi = (lane & O) != 0;
#pragma unroll
        for (int i = 0; i < NV / 2; i++) {
          const float send = hi ? x[i] : x[i + NV / 2];
          const float keep = hi ? x[i + NV / 2] : x[i];
          x[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, O));
        }
        TReduce<NV / 2, O / 2>::run(x, lane);
      } else {
        x[0] = __fadd_rn(x[0], __shfl_xor_sync(0xffffffffu, x[0], O));
        TReduce<1, O / 2>::run(x, lane);
      }
    }
  }
};

// CTA of C holding flattened item x of T (CTA c owns [c*T/C, (c+1)*T/C)).
// floor(num / den) for num >= 0, den > 0: a 32-bit division when both fit
// (the common case), else the 64-bit one
__device__ __forceinline__ long long div_nonneg(long long num, long long den) {
  if (static_cast<unsigned long long>(num | den) <= 0xFFFFFFFFull)
    return static_cast<long long>(static_cast<unsigned>(num) / static_cast<unsigned>(den));
  return num / den;
}
__device__ __forceinline__ int cta_of(long long x, long long T, int C) {
  return static_cast<int>(div_nonneg((x + 1) * C - 1, T));
}

// Item counts of unit u's two slices in a mode (from its validated state).
template <int MODE>
__device__ __forceinline__ void slice_counts(const UnitInfo& inf, int& n0, int& n1) {
  if (MODE == kModeDense) {
    n0 = inf.n;
    n1 = 0;
  } else if (MODE == kModeDet) {
    const int n_extra = inf.mode == 2 ? inf.p : (inf.mode == 1 ? inf.ntail : 0);
    const int n_det = inf.mode == 2 ? inf.nI : inf.nI + n_extra;
    n0 = n_det;
    n1 = inf.nI + n_extra - n_det;
  } else {
    const bool whole_tail = inf.mode == 2 && inf.exhausted;
    const bool sampled = inf.mode == 2 && !inf.exhausted;
    n0 = whole_tail ? inf.ntail : 0;
    n1 = sampled ? inf.bsz - inf.p : 0;
  }
}

// Exclusive prefix over 2*units slice counts into pre[0 .. 2*units] (one CTA).
template <int MODE>
__device__ void write_slice_prefix(const DevParams& P, long long* pre, unsigned* s_warp,
                                   long long* s_carry) {
  if (threadIdx.x == 0) *s_carry = 0;
  __syncthreads();
  const int ns = 2 * P.units;
  for (int base = 0; base < ns; base += blockDim.x) {
    const int sidx = base + threadIdx.x;
    unsigned cnt = 0;
    if (sidx < ns) {
      UnitInfo inf;
      const int4* src = reinterpret_cast<const int4*>(P.info + (sidx >> 1));
      int4* dst = reinterpret_cast<int4*>(&inf);
#pragma unroll
      for (int i = 0; i < static_cast<int>(sizeof(UnitInfo) / 16); i++) dst[i] = __ldcg(src + i);
      int n0, n1;
      slice_counts<MODE>(inf, n0, n1);
      cnt = static_cast<unsigned>((sidx & 1) ? n1 : n0);
    }
    const long long carry = *s_carry;
    const unsigned incl = block_inclusive_scan(cnt, s_warp);  // a 256-slice chunk sum fits in 32 bits
    if (sidx < ns) pre[sidx] = carry + (incl - cnt);
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) *s_carry = carry + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) pre[ns] = *s_carry;
}

// The records of slice s: one from every producer that owns at least one of
// its items (a producer that owns no item writes none). With T >= C every
// producer owns items, so they are the producers [c_first, c_last]; with
// T < C each owns at most one, so they are the owners of the slice's items,
// one per item. Record j of the slice is at index slice_rec(j) + s.
struct SliceRecs {
  long long x0;   // first item of the slice
  int cf;         // first producer (T >= C)
  int n;          // records
  bool per_item;  // T < C
};
__device__ __forceinline__ SliceRecs slice_recs(const long long* pre, int s, long long T, int C) {
  SliceRecs r{pre[s], 0, 0, T < C};
  const long long x1 = pre[s + 1];
  if (x1 <= r.x0) return r;
  if (r.per_item) {
    r.n = static_cast<int>(x1 - r.x0);
  } else {
    r.cf = cta_of(r.x0, T, C);
    r.n = cta_of(x1 - 1, T, C) - r.cf + 1;
  }
  return r;
}
__device__ __forceinline__ int slice_rec(const SliceRecs& r, long long T, int C, int j) {
  return r.per_item ? cta_of(r.x0 + j, T, C) : r.cf + j;
}

// ============================================================ budget
struct U128 {
  unsigned long long lo, hi;
};
__device__ __forceinline__ U128 u128_add(U128 a, U128 b) {
  U128 r;
  r.lo = a.lo + b.lo;
  r.hi = a.hi + b.hi + (r.lo < a.lo ? 1ull : 0ull);
  return r;
}
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ U128 warp_sum_u128(U128 v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    U128 w;
    w.lo = __shfl_xor_sync(0xffffffffu, v.lo, o);
    w.hi = __shfl_xor_sync(0xffffffffu, v.hi, o);
    v = u128_add(v, w);
  }
  return v;
}

// Per query head: m = max true score over I_f and the pilot (s_mh, from the
// unit's det records: the same fp32 scores, so exact); x = vexp(s - m);
// xq = round(x * 2^32); S_f = sum of xq over I_f, S1 and S2 = sums of xq and
// xq^2 over the pilot (integers, so the reduction order does not matter);
// n_h = (z * N_tail * sigma / (eps * D))^2 with sigma^2 = (p S2 - S1^2) /
// (p (p - 1)) and D = S_f + N_tail * S1 / p, in double in a fixed operation
// order. b = max(p, max_h n_h); b >= N_tail takes the whole tail instead.
// Block of up to 1024 threads.
constexpr int kBudgetBatch = 4;  // items per thread whose scores are loaded together
// The first batch of thread t's scores (items t + k * threads, k < kBudgetBatch),
// loaded by the caller before the score maxima are known.
template <int G>
__device__ __forceinline__ void load_budget_batch(const float* ps, int nA, float (&sv)[kBudgetBatch][G]) {
#pragma unroll
  for (int k = 0; k < kBudgetBatch; k++) {
    const int i = static_cast<int>(threadIdx.x) + k * static_cast<int>(blockDim.x);
#pragma unroll
    for (int g = 0; g < G; g++) sv[k][g] = i < nA ? ps[static_cast<size_t>(i) * G + g] : 0.0f;
  }
}
template <int G>
__device__ void unit_budget(const DevParams& P, int u, const UnitInfo& inf, const float* ps,
                            const float* s_mh, const float (&first)[kBudgetBatch][G]) {
  __shared__ unsigned long long s_a[32][G], s_b[32][G];
  __shared__ U128 s_c[32][G];
  __shared__ int s_need[G];
  const int b = u / P.Hkv, h = u % P.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  if (inf.mode != 2) {
    __syncthreads();
    if (tid == 0) {
      const int bsz = inf.mode == 1 ? inf.ntail : 0;
      P.info[u].bsz = bsz;
      P.info[u].exhausted = inf.mode == 1;
      P.info[u].nitems = inf.nI + bsz;
      P.budgets[u] = bsz;
      P.sel_count[u] = inf.nI + bsz;
    }
    if (tid < G) P.head_need[static_cast<size_t>(b) * P.Hq + h * G + tid] = inf.mode == 1 ? inf.ntail : 0;
    __syncthreads();
    return;
  }
  float mh[G];
#pragma unroll
  for (int g = 0; g < G; g++) mh[g] = s_mh[g];
  const int nA = inf.nI + inf.p;
  unsigned long long sf[G], s1[G];
  U128 s2[G];
#pragma unroll
  for (int g = 0; g < G; g++) {
    sf[g] = s1[g] = 0ull;
    s2[g] = U128{0ull, 0ull};
  }
  constexpr int BATCH = kBudgetBatch;
  const int nt = blockDim.x;
  for (int i0 = tid; i0 < nA; i0 += BATCH * nt) {
    float sv[BATCH][G];
    if (i0 == tid) {  // the first batch arrived with the call
#pragma unroll
      for (int k = 0; k < BATCH; k++)
#pragma unroll
        for (int g = 0; g < G; g++) sv[k][g] = first[k][g];
    } else {
#pragma unroll
      for (int k = 0; k < BATCH; k++) {
        const int i = i0 + k * nt;
#pragma unroll
        for (int g = 0; g < G; g++) sv[k][g] = i < nA ? ps[static_cast<size_t>(i) * G + g] : 0.0f;
      }
    }
#pragma unroll
    for (int k = 0; k < BATCH; k++) {
      const int i = i0 + k * nt;
      if (i >= nA) continue;
#pragma unroll
      for (int g = 0; g < G; g++) {
        const float x = vexp(__fsub_rn(sv[k][g], mh[g]));
        const unsigned long long xq = __float2ull_rn(__fmul_rn(x, 4294967296.0f));
        if (i < inf.nI) {
          sf[g] += xq;
        } else {
          s1[g] += xq;
          s2[g] = u128_add(s2[g], U128{xq * xq, __umul64hi(xq, xq)});
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; g++) {
    sf[g] = warp_sum_u64(sf[g]);
    s1[g] = warp_sum_u64(s1[g]);
    s2[g] = warp_sum_u128(s2[g]);
  }
  __syncthreads();
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; g++) {
      s_a[warp][g] = sf[g];
      s_b[warp][g] = s1[g];
      s_c[warp][g] = s2[g];
    }
  }
  __syncthreads();
  if (tid < G) {
    const int g = tid;
    unsigned long long Sf = 0, S1 = 0;
    U128 S2{0ull, 0ull};
    for (int w = 0; w < nw; w++) {
      Sf += s_a[w][g];
      S1 += s_b[w][g];
      S2 = u128_add(S2, s_c[w][g]);
    }
    const unsigned long long p = static_cast<unsigned long long>(inf.p);
    U128 pS2;  // p * S2, exact
    pS2.lo = p * S2.lo;
    pS2.hi = __umul64hi(p, S2.lo) + p * S2.hi;
    const unsigned long long sq_lo = S1 * S1, sq_hi = __umul64hi(S1, S1);
    U128 V;    // p * S2 - S1^2 >= 0
    V.lo = pS2.lo - sq_lo;
    V.hi = pS2.hi - sq_hi - (pS2.lo < sq_lo ? 1ull : 0ull);
    const double Vd = __dadd_rn(__dmul_rn(__ull2double_rn(V.hi), 18446744073709551616.0),
                                __ull2double_rn(V.lo));
    const double pd = static_cast<double>(inf.p);
    const double var = __ddiv_rn(Vd, __dmul_rn(pd, static_cast<double>(inf.p - 1)));
    const double nt = static_cast<double>(inf.ntail);
    const double Dq = __dadd_rn(__ull2double_rn(Sf), __ddiv_rn(__dmul_rn(nt, __ull2double_rn(S1)), pd));
    const double t = __ddiv_rn(__dmul_rn(P.z, nt), __dmul_rn(static_cast<double>(P.eps), Dq));
    const double need = __dmul_rn(__dmul_rn(t, t), var);
    int nh = need >= nt ? inf.ntail : static_cast<int>(ceil(need));
    if (P.guarantee) nh = max(nh, P.num_need[u * G + g]);
    s_need[g] = nh;
    P.head_need[static_cast<size_t>(b) * P.Hq + h * G + g] = nh;
  }
  __syncthreads();
  if (tid == 0) {
    int nmax = 0;
    for (int g = 0; g < G; g++) nmax = max(nmax, s_need[g]);
    int bsz = max(inf.p, nmax);
    int ex = 0;
    if (bsz >= inf.ntail) {
      bsz = inf.ntail;
      ex = 1;
    }
    P.info[u].bsz = bsz;
    P.info[u].exhausted = ex;
    P.info[u].nitems = inf.nI + bsz;
    P.budgets[u] = bsz;
    P.sel_count[u] = inf.nI + bsz;
  }
  __syncthreads();
}

// ============================================================ k_topp
// Top-p selection (the mass-threshold variant of the predicted top-k): for
// each unit, the number kk of highest-ranked middle positions (ranking key
// order, ties to the lower position) whose share of the middle's softmax mass
// under the scaled ranking scores first reaches p = topp_num / topp_den. Mass
// in 2^-32 fixed point, w_j = rint(vexp(fl(r_j c) - max fl(r c)) 2^32), so the
// cut is the exact integer test prefix * den >= num * S. The cut key comes
// from a weighted radix select (digits of 11, 11 and 10 bits; u64 bin masses,
// u128 comparisons); the keys equal to it all weigh the same, so the number
// of them taken is the smallest m with (mass above + m w) * den >= num * S.
// Writes the unit's k (and the regions that follow from it) and its window
// positions; the last CTA then rebuilds the det gather's slice prefix. The
// count-based select that follows takes exactly those kk keys. One CTA per
// unit, keys read from L2 (the score pass wrote them just before).
constexpr int kToppThreads = 1024;

// fp32 value of an order key (inverse of ord_key; -0 comes back as +0).
__device__ __forceinline__ float key_value(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ bool u128_ge(U128 a, U128 b) { return a.hi != b.hi ? a.hi > b.hi : a.lo >= b.lo; }
__device__ __forceinline__ U128 mul_u64(unsigned long long a, unsigned long long b) {
  return U128{a * b, __umul64hi(a, b)};
}

// Inclusive prefix sum of a u64 over the block (blockDim.x a multiple of 32).
__device__ __forceinline__ unsigned long long block_scan_u64(unsigned long long v, unsigned long long* s_w) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) s_w[warp] = v;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = lane < nw ? s_w[lane] : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < nw) s_w[lane] = w;
  }
  __syncthreads();
  const unsigned long long base = warp > 0 ? s_w[warp - 1] : 0ull;
  __syncthreads();
  return v + base;
}

// Over NB weighted bins (masses hm, counts hc), scanned from the top bin down:
// the bin where (base + cumulative mass) * den first reaches target. Adds the
// mass and count of the bins above it to *s_base / *s_cnt and writes the bin.
template <int NB>
__device__ void find_mass_digit(const unsigned long long* hm, const unsigned* hc, unsigned den, U128 target,
                                unsigned long long* s_base, unsigned* s_cnt, int* s_digit,
                                unsigned long long* s_w, unsigned* s_wc) {
  constexpr int PER = NB / kToppThreads > 0 ? NB / kToppThreads : 1;
  const int t = threadIdx.x;
  const bool owns = (t + 1) * PER <= NB;
  const int lo = owns ? NB - (t + 1) * PER : 0;  // bins [lo, lo + PER), scanned downwards
  unsigned long long m = 0;
  unsigned c = 0;
  if (owns)
#pragma unroll
    for (int i = 0; i < PER; i++) {
      m += hm[lo + i];
      c += hc[lo + i];
    }
  const unsigned long long base = *s_base;
  const unsigned cbase = *s_cnt;
  const unsigned long long incl = block_scan_u64(m, s_w);
  const unsigned cincl = block_inclusive_scan(c, s_wc);
  const unsigned long long excl = incl - m;
  const unsigned cexcl = cincl - c;
  __syncthreads();  // every thread read s_base and s_cnt
  if (owns && u128_ge(mul_u64(base + incl, den), target) && !u128_ge(mul_u64(base + excl, den), target)) {
    unsigned long long acc = base + excl;
    unsigned cacc = cbase + cexcl;
    for (int i = PER - 1; i >= 0; i--) {
      if (u128_ge(mul_u64(acc + hm[lo + i], den), target)) {
        *s_digit = lo + i;
        *s_base = acc;
        *s_cnt = cacc;
        break;
      }
      acc += hm[lo + i];
      cacc += hc[lo + i];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kToppThreads, 1) k_topp(DevParams P) {
  __shared__ unsigned long long s_hm[kHist1];
  __shared__ unsigned s_hc[kHist1];
  __shared__ unsigned long long s_w[32];
  __shared__ unsigned s_wc[32];
  __shared__ unsigned long long s_base;
  __shared__ unsigned s_cnt, s_kmax;
  __shared__ int s_digit, s_last;
  __shared__ long long s_carry;
  const int u = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
  grid_dependency_wait();
  const UnitInfo inf = P.info[u];
  const int mlen = inf.wst - inf.s1;
  const unsigned* keys = P.ordk + static_cast<size_t>(u) * P.max_ctx + inf.s1;
  const unsigned num = static_cast<unsigned>(P.topp_num), den = static_cast<unsigned>(P.topp_den);
  int kk = 0;
  if (inf.n > 0 && mlen > 0 && num > 0) {
    // the largest ranking score of the middle
    unsigned mk = 0;
    for (int x = tid; x < mlen; x += nt) mk = max(mk, __ldcg(keys + x));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mk = max(mk, __shfl_xor_sync(0xffffffffu, mk, o));
    if (tid == 0) s_kmax = 0u;
    __syncthreads();
    if ((tid & 31) == 0) atomicMax(&s_kmax, mk);
    __syncthreads();
    const float smax = __fmul_rn(key_value(s_kmax), P.scale);
    auto weight = [&](unsigned key) -> unsigned long long {
      const float x = vexp(__fsub_rn(__fmul_rn(key_value(key), P.scale), smax));
      return __float2ull_rn(__fmul_rn(x, 4294967296.0f));
    };
    // digit 1 masses and counts, and the total mass S
    for (int i = tid; i < kHist1; i += nt) {
      s_hm[i] = 0ull;
      s_hc[i] = 0u;
    }
    if (tid == 0) {
      s_base = 0ull;
      s_cnt = 0u;
      s_digit = 0;
    }
    __syncthreads();
    unsigned long long tot = 0;
    for (int x = tid; x < mlen; x += nt) {
      const unsigned key = __ldcg(keys + x);
      const unsigned long long w = weight(key);
      tot += w;
      atomicAdd(&s_hm[key >> 21], w);
      atomicAdd(&s_hc[key >> 21], 1u);
    }
    const unsigned long long S = block_scan_u64(tot, s_w);  // the last thread holds the total
    __shared__ unsigned long long s_S;
    if (tid == nt - 1) s_S = S;
    __syncthreads();
    const U128 target = mul_u64(s_S, num);
    find_mass_digit<kHist1>(s_hm, s_hc, den, target, &s_base, &s_cnt, &s_digit, s_w, s_wc);
    const unsigned d1 = static_cast<unsigned>(s_digit);
    // digit 2 within bin d1
    for (int i = tid; i < kHist2; i += nt) {
      s_hm[i] = 0ull;
      s_hc[i] = 0u;
    }
    __syncthreads();
    for (int x = tid; x < mlen; x += nt) {
      const unsigned key = __ldcg(keys + x);
      if ((key >> 21) == d1) {
        atomicAdd(&s_hm[(key >> 10) & 2047u], weight(key));
        atomicAdd(&s_hc[(key >> 10) & 2047u], 1u);
      }
    }
    __syncthreads();
    find_mass_digit<kHist2>(s_hm, s_hc, den, target, &s_base, &s_cnt, &s_digit, s_w, s_wc);
    const unsigned pre = d1 << 11 | static_cast<unsigned>(s_digit);
    // digit 3 within (d1, d2)
    for (int i = tid; i < kHist3; i += nt) {
      s_hm[i] = 0ull;
      s_hc[i] = 0u;
    }
    __syncthreads();
    for (int x = tid; x < mlen; x += nt) {
      const unsigned key = __ldcg(keys + x);
      if ((key >> 10) == pre) {
        atomicAdd(&s_hm[key & 1023u], weight(key));
        atomicAdd(&s_hc[key & 1023u], 1u);
      }
    }
    __syncthreads();
    find_mass_digit<kHist3>(s_hm, s_hc, den, target, &s_base, &s_cnt, &s_digit, s_w, s_wc);
    // the cut key: keys above it are all taken; of the tied ones, the fewest
    // (lowest positions first) that reach the target
    if (tid == 0) {
      const unsigned thr = pre << 10 | static_cast<unsigned>(s_digit);
      const unsigned long long wt = weight(thr);
      unsigned lo = 1, hi = s_hc[s_digit];
      while (lo < hi) {
        const unsigned mid = lo + (hi - lo) / 2;
        if (u128_ge(mul_u64(s_base + static_cast<unsigned long long>(mid) * wt, den), target))
          hi = mid;
        else
          lo = mid + 1;
      }
      s_cnt += lo;
    }
    __syncthreads();
    kk = static_cast<int>(s_cnt);
  }
  // the unit's regions with k = kk, and its window positions
  const int ntail = mlen - kk;
  const int nI = inf.s1 + kk + (inf.n - inf.wst);
  if (tid == 0) {
    P.info[u].k = kk;
    P.info[u].ntail = ntail;
    P.info[u].nI = nI;
    P.info[u].nitems = nI;
    P.info[u].mode = ntail == 0 ? 0 : (ntail <= inf.p ? 1 : 2);
  }
  int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx;
  for (int i = tid; i < inf.n - inf.wst; i += nt) sel[inf.s1 + kk + i] = inf.wst + i;
  // the det gather's slice prefix follows from every unit's new state: the
  // last CTA to get here rebuilds it
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(P.gcnt + 1, 1u) == static_cast<unsigned>(P.units - 1);
  __syncthreads();
  if (s_last) {
    __threadfence();
    write_slice_prefix<kModeDet>(P, P.pre_det, s_wc, &s_carry);
  }
  grid_dependents_launch();
}

// Max score per head over unit u's det records (both parts) into s_mh.
// Thread x always reads head x % G (the block size is a multiple of G); the
// per-thread maxima are then reduced per head.
template <int D, int G>
__device__ void det_record_max(const DevParams& P, int u, float* s_mh) {
  constexpr int REC = G * (2 + D);
  __shared__ float s_w[32][G];
  const long long T = P.pre_det[2 * P.units];
  const SliceRecs r0 = slice_recs(P.pre_det, 2 * u, T, P.CD);
  const SliceRecs r1 = slice_recs(P.pre_det, 2 * u + 1, T, P.CD);
  float m = -INFINITY;
  for (int x = threadIdx.x; x < (r0.n + r1.n) * G; x += blockDim.x) {
    const int r = x / G, g = x % G;
    const size_t id = r < r0.n ? static_cast<size_t>(slice_rec(r0, T, P.CD, r) + 2 * u)
                               : static_cast<size_t>(slice_rec(r1, T, P.CD, r - r0.n) + 2 * u + 1);
    m = fmaxf(m, P.rec_det[id * REC + g * (2 + D)]);
  }
#pragma unroll
  for (int o = 16; o >= G; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane < G) s_w[warp][lane] = m;
  __syncthreads();
  if (threadIdx.x < G) {
    float mm = -INFINITY;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); w++) mm = fmaxf(mm, s_w[w][threadIdx.x]);
    s_mh[threadIdx.x] = mm;
  }
  __syncthreads();
}

// out = (A_0 + w A_1) / (L_0 + w L_1) for unit u, head g from its records,
// with part 1 weighted by w = N_tail / b when the tail was sampled (1
// otherwise). The unit's records of both parts (and, for the sample combine,
// of both gathers) form one list; warp x folds entries x, x + warps, ... with
// a running maximum per part, each lane holding D / 32 accumulator elements,
// the loads of a batch of entries issued before they are folded. The warps'
// states are then merged through shared memory. Only the records written in
// this call are read (slice_recs).
constexpr int kCombWarps = 16;

template <int D, int G, int MODE>
__device__ void unit_combine(const DevParams& P, int u, int g) {
  constexpr int REC = G * (2 + D);
  constexpr int PL = D / 32;                      // accumulator elements per lane
  constexpr int NF = MODE == kModeSample ? 4 : 2; // record lists: (part, gather)
  static_assert(PL % 2 == 0, "float2 loads of the accumulators");
  __shared__ float s_acc[2][kCombWarps][D];
  __shared__ float s_ml[2][kCombWarps][2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = static_cast<int>(blockDim.x >> 5);
  const UnitInfo inf = P.info[u];
  const int b = u / P.Hkv, h = u % P.Hkv;
  const bool whole_tail = MODE == kModeSample && inf.mode == 2 && inf.exhausted;
  const bool sampled = MODE == kModeSample && inf.mode == 2 && !inf.exhausted;
  // list f: part f / 2 of the sample (f even) or det (f odd) gather when
  // sampling, else part f of the det / dense gather; the det gather's part-1
  // records (the pilot) are dropped when the whole tail is taken
  const long long Td = P.pre_det[2 * P.units];
  const long long Ts = MODE == kModeSample ? P.pre_samp[2 * P.units] : 0;
  SliceRecs sr[NF];
  int start[NF + 1];
  start[0] = 0;
#pragma unroll
  for (int f = 0; f < NF; f++) {
    const bool smp = MODE == kModeSample && f % 2 == 0;
    const int part = MODE == kModeSample ? f / 2 : f;
    sr[f] = slice_recs(smp ? P.pre_samp : P.pre_det, 2 * u + part, smp ? Ts : Td, smp ? P.CS : P.CD);
    if (MODE == kModeSample && f == 3 && whole_tail) sr[f].n = 0;
    start[f + 1] = start[f] + sr[f].n;
  }
  const int N = start[NF];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f, a0[PL], a1[PL];
#pragma unroll
  for (int c = 0; c < PL; c++) a0[c] = a1[c] = 0.0f;
  constexpr int B = PL > 2 ? 3 : 4;  // entries loaded together, then folded
  for (int j0 = warp; j0 < N; j0 += B * nwarps) {
    float rm[B], rl[B];
    float2 ra[B][PL / 2];
    int rp[B];
#pragma unroll
    for (int k = 0; k < B; k++) {
      const int j = j0 + k * nwarps;  // the same for every lane: branches are warp-uniform
      rm[k] = -INFINITY;
      rl[k] = 0.0f;
      rp[k] = -1;
#pragma unroll
      for (int c = 0; c < PL / 2; c++) ra[k][c] = make_float2(0.0f, 0.0f);
      if (j >= N) continue;
      const float* base = P.rec_det;
      long long id = 0;
#pragma unroll
      for (int f = 0; f < NF; f++) {
        if (j >= start[f] && j < start[f + 1]) {
          const bool smp = MODE == kModeSample && f % 2 == 0;
          const int part = MODE == kModeSample ? f / 2 : f;
          id = slice_rec(sr[f], smp ? Ts : Td, smp ? P.CS : P.CD, j - start[f]) + 2 * u + part;
          base = smp ? P.rec_samp : P.rec_det;
          rp[k] = part;
        }
      }
      const float* q = base + static_cast<size_t>(id) * REC + g * (2 + D);
      rm[k] = q[0];
      rl[k] = q[1];
#pragma unroll
      for (int c = 0; c < PL / 2; c++) ra[k][c] = *reinterpret_cast<const float2*>(q + 2 + lane * PL + 2 * c);
    }
#pragma unroll
    for (int k = 0; k < B; k++) {
      auto fold = [&](float& ms, float& ls, float (&as)[PL]) {
        const float nm = fmaxf(ms, rm[k]);
        const float so = exp_rel(ms, nm), sn = exp_rel(rm[k], nm);
        ls = ls * so + rl[k] * sn;
#pragma unroll
        for (int c = 0; c < PL / 2; c++) {
          as[2 * c] = as[2 * c] * so + ra[k][c].x * sn;
          as[2 * c + 1] = as[2 * c + 1] * so + ra[k][c].y * sn;
        }
        ms = nm;
      };
      if (rp[k] == 0) fold(m0, l0, a0);
      else if (rp[k] == 1) fold(m1, l1, a1);
    }
  }
  const float m[2] = {m0, m1}, l[2] = {l0, l1};
#pragma unroll
  for (int part = 0; part < 2; part++) {
    if (lane == 0) {
      s_ml[part][warp][0] = m[part];
      s_ml[part][warp][1] = l[part];
    }
#pragma unroll
    for (int c = 0; c < PL; c++) s_acc[part][warp][lane * PL + c] = part == 0 ? a0[c] : a1[c];
  }
  __syncthreads();
  const int e = threadIdx.x;
  if (e >= D) return;
  float M[2], L[2], A[2];
#pragma unroll
  for (int part = 0; part < 2; part++) {
    float mx = -INFINITY;
    for (int x = 0; x < nwarps; x++) mx = fmaxf(mx, s_ml[part][x][0]);
    float ls = 0.0f, as = 0.0f;
    for (int x = 0; x < nwarps; x++) {
      const float sc = exp_rel(s_ml[part][x][0], mx);
      ls += s_ml[part][x][1] * sc;
      as += s_acc[part][x][e] * sc;
    }
    M[part] = mx;
    L[part] = ls;
    A[part] = as;
  }
  float w = 1.0f;
  if (sampled) w = static_cast<float>(static_cast<double>(inf.ntail) / static_cast<double>(inf.bsz));
  float* out = P.out + (static_cast<size_t>(b) * P.Hq + h * G + g) * D + e;
  if (inf.n <= 0) {
    *out = 0.0f;
    return;
  }
  const float Mx = fmaxf(M[0], M[1]);
  const float c0 = exp_rel(M[0], Mx), c1 = exp_rel(M[1], Mx);
  *out = (A[0] * c0 + w * (A[1] * c1)) / (L[0] * c0 + w * (L[1] * c1));
}


// ============================================================ k_score_tma
// The exact / Loki score pass for a contiguous cache (one page per sequence,
// so a unit's middle rows are consecutive in memory): every warp streams
// blocks of BLK consecutive rows (8 KB) through a private ring of NS shared-
// memory stages, one bulk copy per block issued NS - 1 blocks ahead, and
// computes each row's dot from shared memory exactly as k_score_rows does
// (the same chunk chains and the same transposed reduction).
template <typename T, int W>
struct ScoreShape {
  static constexpr int E = Elem<T>::kPer16;
  static constexpr int L = W / E;                  // lanes (16-byte chunks) per row
  static constexpr int RPW = 32 / L;               // rows per warp-wide load
  static constexpr int U = L < 8 ? L : 8;          // rows per lane group per step
  static constexpr int ROWS_STEP = RPW * U;
  static constexpr int ROWB = W * static_cast<int>(sizeof(T));
  static constexpr int BLKB = 8192;
  static constexpr int BLK = BLKB / ROWB;          // rows per block
  static constexpr int STEPS = BLK / ROWS_STEP;
  static constexpr int NW = 8, NS = 3;
  static constexpr size_t OFF_BAR = static_cast<size_t>(NW) * NS * BLKB;  // 192 KB of rings
  static constexpr size_t SMEM = OFF_BAR + static_cast<size_t>(NW) * NS * 8;
  static_assert(BLK % ROWS_STEP == 0, "whole steps per block");
};

template <typename T, int W>
__global__ void __launch_bounds__(ScoreShape<T, W>::NW * 32, 1) k_score_tma(DevParams P) {
  using S = ScoreShape<T, W>;
  constexpr int E = S::E, L = S::L, RPW = S::RPW, U = S::U, ROWB = S::ROWB, BLK = S::BLK, NS = S::NS,
                NW = S::NW;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ unsigned s_hist[kHist1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / L, li = lane % L;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR) + warp * NS;
  unsigned char* ring = smem + static_cast<size_t>(warp) * NS * S::BLKB;
  if (lane < NS) mbar_init(&bars[lane], 1);
  for (int i = threadIdx.x; i < kHist1; i += blockDim.x) s_hist[i] = 0u;
  mbar_init_fence();
  __syncthreads();
  grid_dependency_wait();
  const bool loki = P.proxy == kProxyLoki;
  const T* cache = static_cast<const T*>(loki ? P.kp : P.k);
  const float* qsrc = loki ? P.qsel : P.qbar;

  // work split: the first kScoreStatic of the rows in equal contiguous ranges
  // per CTA, the rest in chunks of kScoreChunkBytes handed out by an atomic
  // counter (zeroed by k_prep), so CTAs that stream faster take more of it
  const long long total = P.prefix[P.units];
  const long long tstat = static_cast<long long>(static_cast<double>(total) * kScoreStaticTma);
  constexpr long long kChunk = kScoreChunkBytes / (W * static_cast<long long>(sizeof(T)));
  const long long nchunk = (total - tstat + kChunk - 1) / kChunk;
  __shared__ int s_u;
  __shared__ long long s_chunk;
  unsigned issued = 0;  // blocks this warp issued so far (stage and phase follow from it)
  bool failed = false;
  long long beg = tstat * blockIdx.x / gridDim.x;
  long long end = tstat * (blockIdx.x + 1) / gridDim.x;
  for (;;) {
  if (beg < end) {
  int u = find_unit_block(P.prefix, P.units, beg, &s_u);
  long long cur = beg;
  while (cur < end) {
    while (P.prefix[u + 1] <= cur) u++;
    const long long uend = min(end, P.prefix[u + 1]);
    const UnitInfo inf = P.info[u];
    if (inf.n > 0) {
      const int b = u / P.Hkv, h = u % P.Hkv;
      const int j0 = inf.s1 + static_cast<int>(cur - P.prefix[u]);
      const int nrow = static_cast<int>(uend - cur);
      float q[E];
#pragma unroll
      for (int e = 0; e < E; e++) q[e] = qsrc[static_cast<size_t>(u) * P.D + li * E + e];
      // the sequence's one page: row j of the unit at rows + j * W
      const size_t page = static_cast<size_t>(P.page_table[static_cast<size_t>(b) * P.pps]);
      const T* rows = cache + (page * P.Hkv + h) * P.ps * static_cast<size_t>(W);
      unsigned* ordk = P.ordk + static_cast<size_t>(u) * P.max_ctx;
      const int nblk = (nrow + BLK - 1) / BLK;
      const int nbw = (!failed && warp < nblk) ? (nblk - warp + NW - 1) / NW : 0;  // blocks warp + t * NW
      int nis = 0;
      auto issue = [&](int t) {
        const int r0 = (warp + t * NW) * BLK;
        const int n = min(BLK, nrow - r0);
        const unsigned g = issued + static_cast<unsigned>(t);
        const int st = static_cast<int>(g % NS);
        fence_proxy_async();  // this lane's reads of the stage come before the copy's writes
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars[st], static_cast<unsigned>(n * ROWB));
          bulk_copy_g2s(ring + st * S::BLKB, rows + static_cast<size_t>(j0 + r0) * W,
                        static_cast<unsigned>(n * ROWB), &bars[st]);
        }
        nis++;
      };
#pragma unroll 1
      for (int t = 0; t < NS - 1 && t < nbw; t++) issue(t);
#pragma unroll 1
      for (int t = 0; t < nbw; t++) {
        if (t + NS - 1 < nbw && !failed) issue(t + NS - 1);
        if (t >= nis) continue;  // never issued (only after a failed wait)
        const unsigned g = issued + static_cast<unsigned>(t);
        const int st = static_cast<int>(g % NS);
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[st], (g / NS) & 1u))) {
          if (!failed && lane == 0) atomicOr(P.err, kDevTimeout);
          failed = true;
          drain_ring(bars, NS, issued, t, nis);
        }
        if (failed) continue;
        const unsigned char* sb = ring + st * S::BLKB;
        const int r0 = (warp + t * NW) * BLK;
        const int n = min(BLK, nrow - r0);
#pragma unroll
        for (int step = 0; step < S::STEPS; step++) {
          float a[U];
#pragma unroll
          for (int k = 0; k < U; k++) {
            const int r = step * S::ROWS_STEP + k * RPW + grp;
            const uint4 raw = r < n ? *reinterpret_cast<const uint4*>(sb + r * ROWB + li * 16)
                                    : make_uint4(0u, 0u, 0u, 0u);
            a[k] = chunk_dot<T>(q, raw);
          }
          const float sc = reduce_rows<L, U>(a, li);
          const int r = step * S::ROWS_STEP + reduce_rows_row<L, U>(li) * RPW + grp;
          if ((li % (L / U)) == 0 && r < n) {
            const unsigned o = ord_key(sc);
            ordk[j0 + r0 + r] = o;
            atomicAdd(&s_hist[o >> 21], 1u);
          }
        }
        __syncwarp();  // the stage is free again
      }
      issued += static_cast<unsigned>(nbw);
      flush_hist(s_hist, P.hist + static_cast<size_t>(u) * kHist1);
    }
    cur = uend;
  }
  }
  // next dynamic chunk
  __syncthreads();
  if (threadIdx.x == 0) s_chunk = static_cast<long long>(atomicAdd(P.gcnt, 1u));
  __syncthreads();
  const long long c = s_chunk;
  if (c >= nchunk) break;
  beg = tstat + c * kChunk;
  end = min(total, beg + kChunk);
  }
}

// ============================================================ k_gather
template <typename T, int D, int G, int MODE, bool HOSTKV = false>
__global__ void __launch_bounds__(GatherShape<T, D, G>::NW * 32, 1) k_gather(const __grid_constant__ DevParams P) {
  using S = GatherShape<T, D, G>;
  constexpr int E = S::E, NC = S::NC, LOGNC = S::LOGNC, RPW = S::RPW, UNR = S::UNR, R = S::R;
  constexpr int ROWB = S::ROWB, NW = S::NW, NS = S::NS, V = S::V, LOGV = S::LOGV, NVF = S::NVF,
                REP = S::REP, REC = S::REC;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / NC, c = lane % NC;
  float* s_sc = reinterpret_cast<float*>(smem + S::OFF_SP) + warp * S::WSP;  // [R][G] scores
  float* s_p = s_sc + R * G;                          // [RPW][UNR][G] weights, each stored twice (a pair)
  float* s_mc = s_p + 2 * R * G;                      // [G] maxima, [G] factors
  float* s_ll = reinterpret_cast<float*>(smem + S::OFF_L) + warp * 32 * NVF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR) + warp * NS;
  unsigned char* ring = smem + static_cast<size_t>(warp) * NS * S::BLKB;

  __shared__ int s_first;
  if (lane < NS) mbar_init(&bars[lane], 1);
  if (threadIdx.x == 0) s_first = 0;
  mbar_init_fence();
  __syncthreads();
  grid_dependency_wait();

  // every warp is a record producer: warp gw of W owns items [T*gw/W, T*(gw+1)/W)
  const long long* pre = (MODE == kModeSample) ? P.pre_samp : P.pre_det;
  float* rec = (MODE == kModeSample) ? P.rec_samp : P.rec_det;
  const int W = gridDim.x * NW, gw = blockIdx.x * NW + warp;
  const long long Tt = pre[2 * P.units];
  const long long cbeg = div_nonneg(Tt * (blockIdx.x * NW), W), cend = div_nonneg(Tt * ((blockIdx.x + 1) * NW), W);
  // the CTA's first slice: the one non-empty slice holding item cbeg
  if (cbeg < cend)
    for (int s = threadIdx.x; s < 2 * P.units; s += blockDim.x)
      if (pre[s] <= cbeg && cbeg < pre[s + 1]) s_first = s;
  __syncthreads();
  int sidx = s_first;
  const long long wbeg = div_nonneg(Tt * gw, W), wend = div_nonneg(Tt * (gw + 1), W);
  long long cur = wbeg;
  const T* kc = static_cast<const T*>(P.k);
  const T* vc = static_cast<const T*>(P.v);
  unsigned issued = 0;  // blocks this warp issued in earlier slices (stage and phase follow from it)
  bool failed = false;

  while (cur < wend) {
    while (pre[sidx + 1] <= cur) sidx++;
    const long long send = min(wend, pre[sidx + 1]);
    const int u = sidx >> 1, part = sidx & 1;
    const int lb = static_cast<int>(cur - pre[sidx]), le = static_cast<int>(send - pre[sidx]);
    const int b = u / P.Hkv, h = u % P.Hkv;
    // my chunk of every head's query, the unit's state and, for a contiguous
    // cache, its one page: all loads issued together
    // packed FMAs compute two dot products at once, each half its own fp32
    // chain: for G < 8 two rows (steps k, k + 1) of one head, with each query
    // element stored twice; for G = 8 two heads of one row (fewer registers)
    constexpr bool kPairSteps = G < 8;
    constexpr int QP = kPairSteps ? G : G / 2;
    float2 q2[QP][E];
#pragma unroll
    for (int j = 0; j < QP; j++)
#pragma unroll
      for (int e = 0; e < E; e++) {
        const size_t qrow = static_cast<size_t>(b) * P.Hq + h * G;
        if (kPairSteps) {
          const float qv = Elem<T>::load(P.q, (qrow + j) * D + c * E + e);
          q2[j][e] = make_float2(qv, qv);
        } else {
          q2[j][e] = make_float2(Elem<T>::load(P.q, (qrow + 2 * j) * D + c * E + e),
                                 Elem<T>::load(P.q, (qrow + 2 * j + 1) * D + c * E + e));
        }
      }
    const UnitInfo inf = P.info[u];
    const int pid_c = P.pps == 1 ? P.page_table[static_cast<size_t>(b) * P.pps] : 0;
    const bool valid = inf.n > 0;
    const int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx;
    const bool whole_tail = MODE == kModeSample && inf.mode == 2 && inf.exhausted;
    int n_det = 0;
    if (MODE == kModeDet) {
      int n0, n1;
      slice_counts<kModeDet>(inf, n0, n1);
      n_det = n0;
    }
    float* ps = (MODE == kModeDet && inf.mode == 2) ? P.pscore + static_cast<size_t>(u) * P.max_ctx * G
                                                     : nullptr;
    // item index in the unit's list of local item x of this slice
    auto item_of = [&](int x) -> int {
      const int l = lb + x;
      if (MODE == kModeDense) return l;
      if (MODE == kModeDet) return part == 0 ? l : n_det + l;
      return inf.nI + (whole_tail ? l : inf.p + l);
    };

    float m_run = -INFINITY;  // lane g < G: running maximum of head g
    float l_own[NVF];
    float2 acc[G][E / 2];
#pragma unroll
    for (int j = 0; j < NVF; j++) l_own[j] = 0.0f;
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
      for (int e = 0; e < E / 2; e++) acc[g][e] = make_float2(0.0f, 0.0f);

    const int nitems = valid ? le - lb : 0;
    const int nblk = (nitems + R - 1) / R;
    // this warp's blocks of R consecutive items (none once a wait has failed)
    const int nbw = failed ? 0 : nblk;
    int nis = 0;  // blocks issued in this slice

    // producer side: lane r < R owns row r of a block
    auto pos_of = [&](int t) -> int {
      const int x = t * R + lane;
      if (t >= nbw || lane >= R || x >= nitems) return -1;
      if (MODE == kModeDense) return lb + x;
      const int i = item_of(x);
      if (MODE == kModeDet && part == 0) {  // sinks and window follow from the regions
        if (i < inf.s1) return i;
        if (i >= inf.s1 + inf.k && i < inf.nI) return inf.wst + (i - inf.s1 - inf.k);
      }
      return sel[i];
    };
    auto pid_of = [&](int pos) -> int {
      if (P.pps == 1) return pid_c;
      return pos < 0 ? 0 : P.page_table[static_cast<size_t>(b) * P.pps + page_slot(P, pos)];
    };
    auto issue = [&](int t, int pos, int pid) {
      const unsigned g = issued + static_cast<unsigned>(t);
      const int st = static_cast<int>(g % NS);
      const int nvalid = min(R, nitems - t * R);
      unsigned char* dst = ring + st * S::BLKB;
      fence_proxy_async();
      nis++;
      // row index in the [rows][D] view of the caches; rows adjacent in
      // memory form runs (a lane starts one when its row does not directly
      // follow the previous lane's)
      int row = lane < nvalid ? (pid * P.Hkv + h) * P.ps + (pos - page_slot(P, pos) * P.ps) : 0;
      if constexpr (HOSTKV) {
        // caches in mapped host memory: the warp reads the block's rows with
        // plain 16-byte loads over the host link (eight in flight per lane),
        // stores them into the stage and completes its phase with a plain
        // arrival; rows past the end are zero
        constexpr int VPR = ROWB / 16;
        constexpr int PER = R * VPR / 32;  // vectors of each matrix per lane
        constexpr int CH = PER < 4 ? PER : 4;
#pragma unroll
        for (int i0 = 0; i0 < PER; i0 += CH) {
          uint4 kx[CH], vx[CH];
#pragma unroll
          for (int i = 0; i < CH; i++) {
            const int x = (i0 + i) * 32 + lane, r = x / VPR, cc = x % VPR;
            const int rr = __shfl_sync(0xffffffffu, row, r);
            kx[i] = vx[i] = make_uint4(0u, 0u, 0u, 0u);
            if (r < nvalid) {
              const size_t off = static_cast<size_t>(rr) * D + cc * E;
              kx[i] = ld_gather(kc + off);
              vx[i] = ld_gather(vc + off);
            }
          }
#pragma unroll
          for (int i = 0; i < CH; i++) {
            const int x = (i0 + i) * 32 + lane, r = x / VPR, cc = x % VPR;
            *reinterpret_cast<uint4*>(dst + r * ROWB + cc * 16) = kx[i];
            *reinterpret_cast<uint4*>(dst + (R + r) * ROWB + cc * 16) = vx[i];
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[st]);
        return;
      }
      const int prev = __shfl_up_sync(0xffffffffu, row, 1);
      const bool start = lane < nvalid && (lane == 0 || row != prev + 1);
      const unsigned starts = __ballot_sync(0xffffffffu, start);
      if (__popc(starts) <= R / 4) {
        // few runs: one bulk copy per run; rows past the end get zero V so
        // that their zero weights give exact zeros
        if (lane == 0) mbar_arrive_expect_tx(&bars[st], static_cast<unsigned>(nvalid * 2 * ROWB));
        __syncwarp();
        if (start) {
          const unsigned later = starts & ~((2u << lane) - 1u);  // run starts after mine
          const int stop = later ? __ffs(later) - 1 : nvalid;
          const unsigned bytes = static_cast<unsigned>((stop - lane) * ROWB);
          const size_t off = static_cast<size_t>(row) * D;
          bulk_copy_g2s(dst + lane * ROWB, kc + off, bytes, &bars[st]);
          bulk_copy_g2s(dst + (R + lane) * ROWB, vc + off, bytes, &bars[st]);
        } else if (lane >= nvalid && lane < R) {
          uint4* z = reinterpret_cast<uint4*>(dst + (R + lane) * ROWB);
#pragma unroll
          for (int i = 0; i < ROWB / 16; i++) z[i] = make_uint4(0u, 0u, 0u, 0u);
        }
      } else {
        // scattered rows: four per tensor copy; rows past the end repeat
        // row 0 (finite values under zero weights)
        const int row0v = __shfl_sync(0xffffffffu, row, 0);
        if (lane >= nvalid) row = row0v;
        const int r1 = __shfl_down_sync(0xffffffffu, row, 1);
        const int r2 = __shfl_down_sync(0xffffffffu, row, 2);
        const int r3 = __shfl_down_sync(0xffffffffu, row, 3);
        if (lane == 0) mbar_arrive_expect_tx(&bars[st], static_cast<unsigned>(R * 2 * ROWB));
        __syncwarp();
        if (lane < R && (lane & 3) == 0) {
          gather4_g2s(dst + lane * ROWB, &P.tmk, row, r1, r2, r3, &bars[st]);
          gather4_g2s(dst + (R + lane) * ROWB, &P.tmv, row, r1, r2, r3, &bars[st]);
        }
      }
    };

    // fill the ring; the address pipeline then runs one and two blocks ahead
    // of the issue (page ids for block t + NS - 1, positions for t + NS)
    int posA;
    {
      int posq[NS], pidq[NS - 1];  // loads of the first blocks, issued together
#pragma unroll
      for (int t = 0; t < NS; t++) posq[t] = pos_of(t);
#pragma unroll
      for (int t = 0; t < NS - 1; t++) pidq[t] = pid_of(posq[t]);
#pragma unroll
      for (int t = 0; t < NS - 1; t++)
        if (t < nbw) issue(t, posq[t], pidq[t]);
      posA = posq[NS - 1];
    }
    int pidA = pid_of(posA);
    int posB = pos_of(NS);

#pragma unroll 1
    for (int t = 0; t < nbw; t++) {
      if (t + NS - 1 < nbw && !failed) issue(t + NS - 1, posA, pidA);
      posA = posB;
      pidA = pid_of(posA);
      posB = pos_of(t + NS + 1);

      if (t >= nis) continue;  // never issued (only after a failed wait)
      const unsigned g = issued + static_cast<unsigned>(t);
      const int st = static_cast<int>(g % NS);
      // every lane waits; the warp goes on only if all saw the copies land
      if (!__all_sync(0xffffffffu, mbar_wait(&bars[st], (g / NS) & 1u))) {
        if (!failed && lane == 0) atomicOr(P.err, static_cast<unsigned>(kDevTimeout));
        failed = true;
        drain_ring(bars, NS, issued, t, nis);
      }
      if (failed) continue;
      const unsigned char* kb = ring + st * S::BLKB;
      const unsigned char* vb = kb + R * ROWB;
      const int row0 = t * R;

      // partial dot products of my chunk, all steps and heads
      float sv[V];
      if constexpr (kPairSteps) {
#pragma unroll
        for (int k = 0; k < UNR; k += 2) {
          const uint4 kr0 = *reinterpret_cast<const uint4*>(kb + (k * RPW + grp) * ROWB + c * 16);
          const uint4 kr1 = *reinterpret_cast<const uint4*>(kb + ((k + 1) * RPW + grp) * ROWB + c * 16);
          float kx0[E], kx1[E];
          Elem<T>::unpack(kr0, kx0);
          Elem<T>::unpack(kr1, kx1);
#pragma unroll
          for (int gg = 0; gg < G; gg++) {
            float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int e = 0; e < E; e++) a = __ffma2_rn(q2[gg][e], make_float2(kx0[e], kx1[e]), a);
            sv[k * G + gg] = a.x;
            sv[(k + 1) * G + gg] = a.y;
          }
        }
      } else {
#pragma unroll
        for (int k = 0; k < UNR; k++) {
          const uint4 kr = *reinterpret_cast<const uint4*>(kb + (k * RPW + grp) * ROWB + c * 16);
          float kx[E];
          Elem<T>::unpack(kr, kx);
#pragma unroll
          for (int j = 0; j < QP; j++) {
            float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int e = 0; e < E; e++) a = __ffma2_rn(q2[j][e], make_float2(kx[e], kx[e]), a);
            sv[k * G + 2 * j] = a.x;
            sv[k * G + 2 * j + 1] = a.y;
          }
        }
      }
      TReduce<V, NC / 2>::run(sv, lane);

      // scores I own: value v = step * G + head
      const bool primary = REP == 1 || (c & (REP - 1)) == 0;
      float s_own[NVF];
#pragma unroll
      for (int j = 0; j < NVF; j++) {
        const int v = LOGV >= LOGNC ? c * NVF + j : (c >> (LOGNC - LOGV));
        const int k = v / G, gg = v % G, r = k * RPW + grp;
        const bool ok = row0 + r < nitems;
        s_own[j] = ok ? __fmul_rn(sv[j], P.scale) : -INFINITY;
        if (primary) {
          s_sc[r * G + gg] = s_own[j];
          if (ps != nullptr && ok) ps[static_cast<size_t>(item_of(row0 + r)) * G + gg] = s_own[j];
        }
      }
      __syncwarp();
      if (lane < G) {
        float bm = -INFINITY;
#pragma unroll
        for (int r = 0; r < R; r++) bm = fmaxf(bm, s_sc[r * G + lane]);
        const float mn = fmaxf(m_run, bm);
        s_mc[lane] = mn;
        s_mc[G + lane] = exp_rel(m_run, mn);
        m_run = mn;
      }
      __syncwarp();
      float cf[G];
      bool resc = false;
#pragma unroll
      for (int gg = 0; gg < G; gg++) {
        cf[gg] = s_mc[G + gg];
        resc |= cf[gg] != 1.0f;
      }
      if (resc) {  // the same for every lane
#pragma unroll
        for (int gg = 0; gg < G; gg++)
#pragma unroll
          for (int e = 0; e < E / 2; e++) {
            acc[gg][e].x *= cf[gg];
            acc[gg][e].y *= cf[gg];
          }
      }
#pragma unroll
      for (int j = 0; j < NVF; j++) {
        const int v = LOGV >= LOGNC ? c * NVF + j : (c >> (LOGNC - LOGV));
        const int k = v / G, gg = v % G;  // gg depends on the lane: read its (m, cf) from shared memory
        const float pj = s_own[j] == -INFINITY ? 0.0f : __expf(s_own[j] - s_mc[gg]);
        if (primary) {
          l_own[j] = l_own[j] * s_mc[G + gg] + pj;
          reinterpret_cast<float2*>(s_p)[(grp * UNR + k) * G + gg] = make_float2(pj, pj);
        }
      }
      __syncwarp();
      // value accumulation: my chunk of each of my rows, every head
#pragma unroll
      for (int k = 0; k < UNR; k++) {
        float2 pw[G];
        const float2* pk = reinterpret_cast<const float2*>(s_p) + (grp * UNR + k) * G;
        if constexpr (G % 2 == 0) {
#pragma unroll
          for (int gg = 0; gg < G; gg += 2) {
            const float4 w4 = *reinterpret_cast<const float4*>(pk + gg);
            pw[gg] = make_float2(w4.x, w4.y);
            pw[gg + 1] = make_float2(w4.z, w4.w);
          }
        } else {
          pw[0] = pk[0];
        }
        const uint4 vr = *reinterpret_cast<const uint4*>(vb + (k * RPW + grp) * ROWB + c * 16);
        float vx[E];
        Elem<T>::unpack(vr, vx);
#pragma unroll
        for (int gg = 0; gg < G; gg++)
#pragma unroll
          for (int e = 0; e < E / 2; e++)
            acc[gg][e] = __ffma2_rn(pw[gg], make_float2(vx[2 * e], vx[2 * e + 1]), acc[gg][e]);
      }
      __syncwarp();  // the stage and the score buffers are free again
    }
    issued += static_cast<unsigned>(nbw);

    // ---- this warp's record for the slice: (m, l, acc[D]) per head
#pragma unroll
    for (int o = NC; o < 32; o <<= 1)
#pragma unroll
      for (int gg = 0; gg < G; gg++)
#pragma unroll
        for (int e = 0; e < E / 2; e++) {
          acc[gg][e].x += __shfl_xor_sync(0xffffffffu, acc[gg][e].x, o);
          acc[gg][e].y += __shfl_xor_sync(0xffffffffu, acc[gg][e].y, o);
        }
#pragma unroll
    for (int j = 0; j < NVF; j++) s_ll[lane * NVF + j] = l_own[j];
    __syncwarp();
    float* r = rec + static_cast<size_t>(gw + sidx) * REC;
    if (lane < G) {
      float lsum = 0.0f;
      for (int x = 0; x < 32 * NVF; x++) {
        const int ln = x / NVF, j = x % NVF, cc = ln % NC;
        const int v = LOGV >= LOGNC ? cc * NVF + j : (cc >> (LOGNC - LOGV));
        if (v % G == lane) lsum += s_ll[x];
      }
      r[lane * (2 + D)] = m_run;
      r[lane * (2 + D) + 1] = lsum;
    }
    if (grp == 0) {
#pragma unroll
      for (int gg = 0; gg < G; gg++)
#pragma unroll
        for (int e = 0; e < E / 2; e++) {
          r[gg * (2 + D) + 2 + c * E + 2 * e] = acc[gg][e].x;
          r[gg * (2 + D) + 2 + c * E + 2 * e + 1] = acc[gg][e].y;
        }
    }
    __syncwarp();  // s_ll is reused by the next slice
    cur = send;
  }
  grid_dependents_launch();
}

// ============================================================ k_gather_tc
// The sample and dense gathers for bf16 caches in device memory, on the
// tensor cores. The streaming scheme is k_gather's (persistent grid, every
// warp a record producer over a contiguous item range, a private ring of
// stages filled NS - 1 blocks ahead, bounded mbarrier waits), but every row
// arrives through tile::gather4 copies of 128-byte half rows with the 128-byte
// swizzle (the 16-byte chunk index within a half row XORed with the row's
// index mod 8), so the fragment loads of eight rows touch eight different
// bank groups. Per block of 16 rows: the scores S[r][g] = K[r] . q_g as
// D / 16 bf16 MMAs (m16n8k16, the group's heads in the 8 columns, fp32
// accumulation), the online softmax in the accumulator layout (each lane holds
// heads 2 (lane % 4) and 2 (lane % 4) + 1 of rows lane / 4 and lane / 4 + 8),
// then O^T[d][g] += V^T[d][r] P[r][g] as D / 16 MMAs per term of the weights
// split into two bf16 terms (hi = bf16(p), lo = bf16(p - hi): 2^-16 relative),
// the weights' fragment transposed into the operand layout by movmatrix. The
// output accumulator has the same columns as the scores, so rescaling by a new
// running maximum needs no exchange between lanes. The records are
// k_gather's: (m, l, acc[D]) per head.
template <int D, int G>
struct TcShape {
  static constexpr int R = 16;                     // rows per block
  static constexpr int H = D / 64;                 // 128-byte halves of a row
  static constexpr int HALF = R * 128;             // bytes of one half of a block's rows
  static constexpr int MATB = H * HALF;            // the block's K (or V) rows
  static constexpr int BLKB = 2 * MATB;            // K, then V
  static constexpr int NW = 8;                     // warps per CTA
  static constexpr int NS = (192 * 1024) / (NW * BLKB);  // stages filling a 192 KB ring
  static constexpr int KT = D / 16;                // k-steps of a score tile; M-tiles of the output
  static constexpr int REC = G * (2 + D);
  static constexpr size_t RING = static_cast<size_t>(NW) * NS * BLKB;
  static constexpr size_t OFF_BAR = RING;
  static constexpr size_t SMEM = 1024 + OFF_BAR + static_cast<size_t>(NW) * NS * 8;  // 1 KB to align the ring
  static_assert(G <= 8, "the group's heads fit the 8 columns of a score tile");
  static_assert(D % 64 == 0, "whole 128-byte half rows");
  static_assert(SMEM <= 227 * 1024, "tensor-core gather shared memory");
};

// Byte offset of 16-byte chunk ch of row r in a swizzled [16 rows][D] bf16
// tile (halves of 16 x 128 bytes, 1024-byte aligned).
__device__ __forceinline__ unsigned tc_off(int r, int ch) {
  return static_cast<unsigned>((ch >> 3) * (16 * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}
__device__ __forceinline__ void ldsm_x4(unsigned addr, unsigned (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(unsigned addr, unsigned (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ unsigned movm_t(unsigned x) {
  unsigned y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const unsigned (&a)[4], unsigned b0, unsigned b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// two floats as bf16 (first in the low half), rounded to nearest
__device__ __forceinline__ unsigned pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const unsigned*>(&v);
}
// (hi, lo) bf16 terms of two weights: p = hi + lo to 2^-16 relative
__device__ __forceinline__ void split_bf16x2(float p0, float p1, unsigned& hi, unsigned& lo) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
  hi = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
  lo = pack_bf16x2(p0 - __bfloat162float(h0), p1 - __bfloat162float(h1));
}
// tile::gather4 copy of four rows' columns [x, x + box) into shared memory
__device__ __forceinline__ void gather4x_g2s(void* dst, const CUtensorMap* map, int x, int y0, int y1, int y2,
                                             int y3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}

template <int D, int G, int MODE>
__global__ void __launch_bounds__(TcShape<D, G>::NW * 32, 1) k_gather_tc(const __grid_constant__ DevParams P) {
  using S = TcShape<D, G>;
  constexpr int R = S::R, H = S::H, HALF = S::HALF, MATB = S::MATB, BLKB = S::BLKB, NW = S::NW, NS = S::NS,
                KT = S::KT, REC = S::REC;
  static_assert(MODE == kModeSample || MODE == kModeDense, "sample and dense gathers");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR) + warp * NS;
  unsigned char* ring = smem + static_cast<size_t>(warp) * NS * BLKB;
  const unsigned ring_s = smem_u32(ring);

  __shared__ int s_first;
  if (lane < NS) mbar_init(&bars[lane], 1);
  if (threadIdx.x == 0) s_first = 0;
  mbar_init_fence();
  __syncthreads();
  grid_dependency_wait();

  // every warp is a record producer: warp gw of W owns items [T*gw/W, T*(gw+1)/W)
  const long long* pre = (MODE == kModeSample) ? P.pre_samp : P.pre_det;
  float* rec = (MODE == kModeSample) ? P.rec_samp : P.rec_det;
  const int W = gridDim.x * NW, gw = blockIdx.x * NW + warp;
  const long long Tt = pre[2 * P.units];
  const long long cbeg = div_nonneg(Tt * (blockIdx.x * NW), W), cend = div_nonneg(Tt * ((blockIdx.x + 1) * NW), W);
  if (cbeg < cend)
    for (int s = threadIdx.x; s < 2 * P.units; s += blockDim.x)
      if (pre[s] <= cbeg && cbeg < pre[s + 1]) s_first = s;
  __syncthreads();
  int sidx = s_first;
  const long long wbeg = div_nonneg(Tt * gw, W), wend = div_nonneg(Tt * (gw + 1), W);
  long long cur = wbeg;
  unsigned issued = 0;  // blocks this warp issued in earlier slices (stage and phase follow from it)
  bool failed = false;
  // fragment addresses: lane i serves matrix i / 8, row i % 8 of an ldmatrix.x4
  const int fj = lane >> 3, fr = lane & 7;
  const int hc = 2 * (lane & 3);  // this lane's two head columns

  while (cur < wend) {
    while (pre[sidx + 1] <= cur) sidx++;
    const long long send = min(wend, pre[sidx + 1]);
    const int u = sidx >> 1;
    const int lb = static_cast<int>(cur - pre[sidx]), le = static_cast<int>(send - pre[sidx]);
    const int b = u / P.Hkv, h = u % P.Hkv;
    // the query operand: B[k = d][n = head] = q_head[d]; lane holds head lane / 4,
    // dims 16 kt + 2 (lane % 4) + {0, 1} and those + 8 (zero columns past G)
    unsigned qf[KT][2];
    {
      const int qh = lane >> 2;
      const unsigned short* qp = static_cast<const unsigned short*>(P.q) +
                                 (static_cast<size_t>(b) * P.Hq + h * G + (qh < G ? qh : 0)) * D + hc;
#pragma unroll
      for (int kt = 0; kt < KT; kt++)
#pragma unroll
        for (int x = 0; x < 2; x++) {
          const unsigned lo = qp[16 * kt + 8 * x], hi = qp[16 * kt + 8 * x + 1];
          qf[kt][x] = qh < G ? (lo | (hi << 16)) : 0u;
        }
    }
    const UnitInfo inf = P.info[u];
    const int pid_c = P.pps == 1 ? P.page_table[static_cast<size_t>(b) * P.pps] : 0;
    const bool valid = inf.n > 0;
    const int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx;
    const bool whole_tail = MODE == kModeSample && inf.mode == 2 && inf.exhausted;

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
    float o[KT][4];
#pragma unroll
    for (int mt = 0; mt < KT; mt++)
#pragma unroll
      for (int x = 0; x < 4; x++) o[mt][x] = 0.0f;

    const int nitems = valid ? le - lb : 0;
    const int nblk = (nitems + R - 1) / R;
    const int nbw = failed ? 0 : nblk;
    int nis = 0;  // blocks issued in this slice

    // producer side: lane r < R owns row r of a block
    auto pos_of = [&](int t) -> int {
      const int x = t * R + lane;
      if (t >= nbw || lane >= R || x >= nitems) return -1;
      if (MODE == kModeDense) return lb + x;
      return sel[inf.nI + (whole_tail ? lb + x : inf.p + lb + x)];
    };
    auto pid_of = [&](int pos) -> int {
      if (P.pps == 1) return pid_c;
      return pos < 0 ? 0 : P.page_table[static_cast<size_t>(b) * P.pps + page_slot(P, pos)];
    };
    auto issue = [&](int t, int pos, int pid) {
      const unsigned g = issued + static_cast<unsigned>(t);
      const int st = static_cast<int>(g % NS);
      const int nvalid = min(R, nitems - t * R);
      unsigned char* dst = ring + st * BLKB;
      fence_proxy_async();
      nis++;
      // rows past the end repeat row 0 (finite values under zero weights)
      int row = lane < nvalid ? (pid * P.Hkv + h) * P.ps + (pos - page_slot(P, pos) * P.ps) : 0;
      const int row0v = __shfl_sync(0xffffffffu, row, 0);
      if (lane >= nvalid) row = row0v;
      const int r1 = __shfl_down_sync(0xffffffffu, row, 1);
      const int r2 = __shfl_down_sync(0xffffffffu, row, 2);
      const int r3 = __shfl_down_sync(0xffffffffu, row, 3);
      if (lane == 0) mbar_arrive_expect_tx(&bars[st], static_cast<unsigned>(BLKB));
      __syncwarp();
      if (lane < R && (lane & 3) == 0) {
#pragma unroll
        for (int hf = 0; hf < H; hf++) {
          gather4x_g2s(dst + hf * HALF + lane * 128, &P.tmk_sw, hf * 64, row, r1, r2, r3, &bars[st]);
          gather4x_g2s(dst + MATB + hf * HALF + lane * 128, &P.tmv_sw, hf * 64, row, r1, r2, r3, &bars[st]);
        }
      }
    };

    // fill the ring; the address pipeline then runs one and two blocks ahead
    // of the issue (page ids for block t + NS - 1, positions for t + NS)
    int posA;
    {
      int posq[NS], pidq[NS - 1];
#pragma unroll
      for (int t = 0; t < NS; t++) posq[t] = pos_of(t);
#pragma unroll
      for (int t = 0; t < NS - 1; t++) pidq[t] = pid_of(posq[t]);
#pragma unroll
      for (int t = 0; t < NS - 1; t++)
        if (t < nbw) issue(t, posq[t], pidq[t]);
      posA = posq[NS - 1];
    }
    int pidA = pid_of(posA);
    int posB = pos_of(NS);

#pragma unroll 1
    for (int t = 0; t < nbw; t++) {
      if (t + NS - 1 < nbw && !failed) issue(t + NS - 1, posA, pidA);
      posA = posB;
      pidA = pid_of(posA);
      posB = pos_of(t + NS + 1);

      if (t >= nis) continue;  // never issued (only after a failed wait)
      const unsigned g = issued + static_cast<unsigned>(t);
      const int st = static_cast<int>(g % NS);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars[st], (g / NS) & 1u))) {
        if (!failed && lane == 0) atomicOr(P.err, static_cast<unsigned>(kDevTimeout));
        failed = true;
        drain_ring(bars, NS, issued, t, nis);
      }
      if (failed) continue;
      const unsigned kb = ring_s + static_cast<unsigned>(st * BLKB), vb = kb + MATB;

      // scores: S[r][head] over D / 16 k-steps
      float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int kt = 0; kt < KT; kt++) {
        unsigned a[4];
        ldsm_x4(kb + tc_off(((fj & 1) << 3) | fr, 2 * kt + (fj >> 1)), a);
        mma_bf16(sc, a, qf[kt][0], qf[kt][1]);
      }
      // online softmax: rows lane / 4 (values 0, 1) and lane / 4 + 8 (2, 3)
      const int nvalid = min(R, nitems - t * R);
      const int ra = lane >> 2;
      float sv[4];
#pragma unroll
      for (int x = 0; x < 4; x++) sv[x] = (ra + (x >> 1) * 8) < nvalid ? sc[x] * P.scale : -INFINITY;
      float bm[2] = {fmaxf(sv[0], sv[2]), fmaxf(sv[1], sv[3])};
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)
#pragma unroll
        for (int k = 0; k < 2; k++) bm[k] = fmaxf(bm[k], __shfl_xor_sync(0xffffffffu, bm[k], off));
      float cf[2];
#pragma unroll
      for (int k = 0; k < 2; k++) {
        const float nm = fmaxf(m_run[k], bm[k]);
        cf[k] = exp_rel(m_run[k], nm);
        m_run[k] = nm;
      }
      float pv[4];
#pragma unroll
      for (int x = 0; x < 4; x++) pv[x] = sv[x] == -INFINITY ? 0.0f : __expf(sv[x] - m_run[x & 1]);
#pragma unroll
      for (int k = 0; k < 2; k++) l_run[k] = l_run[k] * cf[k] + (pv[k] + pv[2 + k]);
      if (__any_sync(0xffffffffu, cf[0] != 1.0f || cf[1] != 1.0f)) {
#pragma unroll
        for (int mt = 0; mt < KT; mt++)
#pragma unroll
          for (int x = 0; x < 4; x++) o[mt][x] *= cf[x & 1];
      }
      // the weights as the B operand B[k = r][n = head]: transposes of the
      // [r][head-pair] fragments of rows 0-7 and 8-15
      unsigned ph0, pl0, ph1, pl1;
      split_bf16x2(pv[0], pv[1], ph0, pl0);
      split_bf16x2(pv[2], pv[3], ph1, pl1);
      ph0 = movm_t(ph0);
      pl0 = movm_t(pl0);
      ph1 = movm_t(ph1);
      pl1 = movm_t(pl1);
      // O^T[d][head] += V^T[d][r] P[r][head], one M-tile of 16 dims at a time
#pragma unroll
      for (int mt = 0; mt < KT; mt++) {
        unsigned a[4];
        ldsm_x4_t(vb + tc_off(((fj >> 1) << 3) | fr, 2 * mt + (fj & 1)), a);
        mma_bf16(o[mt], a, ph0, ph1);
        mma_bf16(o[mt], a, pl0, pl1);
      }
      __syncwarp();  // the stage is free again
    }
    issued += static_cast<unsigned>(nbw);

    // ---- this warp's record for the slice: (m, l, acc[D]) per head; lane
    // holds dims 16 mt + lane / 4 (+ 8) of heads hc, hc + 1
#pragma unroll
    for (int off = 4; off < 32; off <<= 1)
#pragma unroll
      for (int k = 0; k < 2; k++) l_run[k] += __shfl_xor_sync(0xffffffffu, l_run[k], off);
    float* r = rec + static_cast<size_t>(gw + sidx) * REC;
#pragma unroll
    for (int k = 0; k < 2; k++) {
      const int hh = hc + k;
      if (hh >= G) continue;
      float* rh = r + hh * (2 + D);
      if (lane < 4) {
        rh[0] = m_run[k];
        rh[1] = l_run[k];
      }
#pragma unroll
      for (int mt = 0; mt < KT; mt++) {
        rh[2 + 16 * mt + (lane >> 2)] = o[mt][k];
        rh[2 + 16 * mt + (lane >> 2) + 8] = o[mt][2 + k];
      }
    }
    __syncwarp();
    cur = send;
  }

  grid_dependents_launch();
}

// ============================================================ draw positions
// Cache positions of unit u's sampled entries t in [t0, t1): with a sampled
// tail, draw t is the Lemire map of Philox word t onto the tail; when the tail
// is taken whole, entry t is the t-th tail position. Written to
// sel[nI + t]. The sorted top-k list is staged in s_topk when it fits.
__device__ void write_draw_positions(const DevParams& P, int u, const UnitInfo& inf, bool whole_tail,
                                     int t0, int t1, int* s_topk) {
  const int* g = P.sel + static_cast<size_t>(u) * P.max_ctx + inf.s1;
  const int* topk = g;
  if (inf.k <= kTopkSmem) {
    for (int x = threadIdx.x; x < inf.k; x += blockDim.x) s_topk[x] = g[x];
    __syncthreads();
    topk = s_topk;
  }
  int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx + inf.nI;
  // the draw counter names the sequence and KV head in the whole batch (a
  // shard adds its offsets), so a shard draws what the whole batch would
  const unsigned bb = static_cast<unsigned>(P.batch_offset + u / P.Hkv),
                 hh = static_cast<unsigned>(P.head_offset + u % P.Hkv);
  const int step0 = inf.k > 0 ? 1 << (31 - __clz(inf.k)) : 0;
  // each thread takes aligned groups of four draws: one Philox block serves
  // all four, and their four searches advance together
  for (int t4 = (t0 & ~3) + 4 * static_cast<int>(threadIdx.x); t4 < t1; t4 += 4 * static_cast<int>(blockDim.x)) {
    int rho[4];
    if (whole_tail) {
#pragma unroll
      for (int j = 0; j < 4; j++) rho[j] = t4 + j;
    } else {
      const uint4 q = draw_block(P.seed, bb, hh, static_cast<unsigned>(t4) >> 2);
      rho[0] = lemire(q.x, inf.ntail);
      rho[1] = lemire(q.y, inf.ntail);
      rho[2] = lemire(q.z, inf.ntail);
      rho[3] = lemire(q.w, inf.ntail);
    }
    // c_j = #{i : topk[i] - s1 - i <= rho_j} by binary lifting (the left side
    // is non-decreasing in i)
    int c[4] = {0, 0, 0, 0};
    for (int step = step0; step > 0; step >>= 1) {
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const int i = c[j] + step;
        if (i <= inf.k && topk[i - 1] - inf.s1 - (i - 1) <= rho[j]) c[j] = i;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const int t = t4 + j;
      if (t >= t0 && t < t1) sel[t] = inf.s1 + rho[j] + c[j];
    }
  }
  __syncthreads();
}

// ============================================================ k_topk
// Top-k selection and pilot draws of one unit in one CTA (kTopkThreadsFew or
// kTopkThreads threads), for any middle length. The keys are read from L2 (the score pass wrote them just
// before) in one ordered pass: digit 1 (key bits 31..21) of the k-th largest
// key comes from the score pass's histogram; each warp turns 1024 consecutive
// keys per round into 32 words of two ballots (key above bin d1; key in bin
// d1), and a block scan over the packed popcounts appends the positions of
// both kinds to shared-memory lists in position order, while the keys of bin
// d1 are counted by digit 2. Every key above bin d1 is in the top k. Digit 3
// and the threshold key then come from the bin-d1 list alone; its members
// above the threshold, and the lowest-positioned ones equal to it, are
// compacted in order, and the two ascending lists are merged into sel (and
// into shared memory for the draws). When a list would overflow its space
// (e.g. every score equal), a second ordered pass over all keys selects
// instead. Then the pilot draws (or the whole tail when it is no larger than
// the pilot), as k_draws does for the sample.
// threads per CTA: 1024 when every unit has an SM of its own, else 512 (two CTAs per SM)
constexpr int kTopkThreadsFew = 1024, kTopkThreads = 512;
constexpr int kTopkAbove = 4096;   // positions above bin d1 kept in shared memory
constexpr int kTopkCand = 8192;    // positions in bin d1
constexpr int kTopkTaken = 4096;   // bin-d1 positions taken
constexpr int kTopkList = 6144;    // the merged list, kept for the draws
constexpr size_t kTopkKernelSmem = static_cast<size_t>(kHist2 + kTopkAbove + kTopkCand + kTopkTaken + kTopkList) * 4;

// Position of v among n ascending values (the count of those below it).
__device__ __forceinline__ int lower_bound_s(const int* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

template <int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) k_topk(DevParams P) {
  extern __shared__ __align__(16) unsigned char topk_smem[];
  unsigned* s_hist = reinterpret_cast<unsigned*>(topk_smem);  // [kHist2]
  int* s_above = reinterpret_cast<int*>(s_hist + kHist2);     // [kTopkAbove]
  int* s_cand = s_above + kTopkAbove;                         // [kTopkCand]
  int* s_took = s_cand + kTopkCand;                           // [kTopkTaken]
  int* s_list = s_took + kTopkTaken;                          // [kTopkList]
  __shared__ unsigned s_warp[32];
  __shared__ int s_digit, s_krem;
  __shared__ unsigned s_round[2];
  constexpr int NWK = NT / 32;
  const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_dependency_wait();
  const UnitInfo inf = P.info[u];
  const int* topk = P.sel + static_cast<size_t>(u) * P.max_ctx + inf.s1;  // global copy
  if (inf.k > 0) {
    const int mlen = inf.wst - inf.s1, k = inf.k;
    const unsigned* keys = P.ordk + static_cast<size_t>(u) * P.max_ctx + inf.s1;
    int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx + inf.s1;
    const bool keep = k <= kTopkList;
    // digit 1 from the score pass's histogram
    const unsigned* h1 = P.hist + static_cast<size_t>(u) * kHist1;
    for (int x = tid; x < kHist1; x += NT) s_hist[x] = __ldcg(h1 + x);
    if (tid == 0) {
      s_digit = 0;
      s_krem = k;
    }
    __syncthreads();
    find_digit_bt<kHist1, NT>(s_hist, k, &s_digit, &s_krem, s_warp);
    const unsigned d1 = static_cast<unsigned>(s_digit);
    const int krem1 = s_krem;
    for (int x = tid; x < kHist2; x += NT) s_hist[x] = 0u;
    __syncthreads();

    // one ordered pass: positions above bin d1, positions in it, digit-2 counts
    unsigned na = 0, nc = 0;
    for (int base = 0; base < mlen; base += 1024 * NWK) {
      const int wb = base + warp * 1024;
      unsigned wa = 0, wc = 0;
#pragma unroll
      for (int half = 0; half < 2; half++) {
        unsigned o[16];
#pragma unroll
        for (int i = 0; i < 16; i++) {
          const int x = wb + (half * 16 + i) * 32 + lane;
          o[i] = x < mlen ? __ldcg(keys + x) : 0u;
        }
#pragma unroll
        for (int i = 0; i < 16; i++) {
          const int x = wb + (half * 16 + i) * 32 + lane;
          const unsigned dg = o[i] >> 21;
          const bool in = x < mlen && dg == d1;
          const unsigned ba = __ballot_sync(0xffffffffu, x < mlen && dg > d1);
          const unsigned bc = __ballot_sync(0xffffffffu, in);
          if (in) atomicAdd(&s_hist[(o[i] >> 10) & 2047u], 1u);
          if (lane == half * 16 + i) {
            wa = ba;
            wc = bc;
          }
        }
      }
      // a round holds at most 1024 * NWK keys, so both counts fit 16 bits
      const unsigned packed = (static_cast<unsigned>(__popc(wa)) << 16) | static_cast<unsigned>(__popc(wc));
      const unsigned incl = block_inclusive_scan(packed, s_warp);
      const unsigned excl = incl - packed;
      unsigned pa = na + (excl >> 16), pc = nc + (excl & 0xFFFFu);
      for (unsigned m = wa; m; m &= m - 1u, pa++)
        if (pa < static_cast<unsigned>(kTopkAbove)) s_above[pa] = wb + lane * 32 + (__ffs(m) - 1);
      for (unsigned m = wc; m; m &= m - 1u, pc++)
        if (pc < static_cast<unsigned>(kTopkCand)) s_cand[pc] = wb + lane * 32 + (__ffs(m) - 1);
      if (tid == NT - 1) {
        s_round[0] = incl >> 16;
        s_round[1] = incl & 0xFFFFu;
      }
      __syncthreads();
      na += s_round[0];
      nc += s_round[1];
      __syncthreads();
    }
    // digit 2
    find_digit_bt<kHist2, NT>(s_hist, krem1, &s_digit, &s_krem, s_warp);
    const unsigned pre = d1 << 11 | static_cast<unsigned>(s_digit);
    const int krem2 = s_krem;
    // digit 3 over the bin-d1 list (over every key when it overflowed)
    for (int x = tid; x < kHist3; x += NT) s_hist[x] = 0u;
    __syncthreads();
    const bool cand_ok = nc <= static_cast<unsigned>(kTopkCand);
    // the candidates' keys, kept for the compaction in s_list (unused until
    // the merge) when they fit
    unsigned* s_ckey = reinterpret_cast<unsigned*>(s_list);
    const bool ckey = nc <= static_cast<unsigned>(kTopkList);
    if (cand_ok) {
      for (int i = tid; i < static_cast<int>(nc); i += NT) {
        const unsigned o = __ldcg(keys + s_cand[i]);
        if (ckey) s_ckey[i] = o;
        if ((o >> 10) == pre) atomicAdd(&s_hist[o & 1023u], 1u);
      }
    } else {
      for (int x = tid; x < mlen; x += NT) {
        const unsigned o = __ldcg(keys + x);
        if ((o >> 10) == pre) atomicAdd(&s_hist[o & 1023u], 1u);
      }
    }
    __syncthreads();
    find_digit_bt<kHist3, NT>(s_hist, krem2, &s_digit, &s_krem, s_warp);
    const unsigned thr = pre << 10 | static_cast<unsigned>(s_digit);
    const unsigned need_eq = static_cast<unsigned>(s_krem);
    if (tid == 0) {
      P.info[u].thr = thr;
      P.info[u].need_eq = static_cast<int>(need_eq);
    }
    const int ntake = k - static_cast<int>(na);  // bin-d1 members taken
    if (cand_ok && na <= static_cast<unsigned>(kTopkAbove) && ntake >= 0 && ntake <= kTopkTaken) {
      // the bin-d1 members taken, in position order: every one above thr, and
      // the first need_eq equal to it
      unsigned eq_seen = 0, taken = 0;
      for (int base = 0; base < static_cast<int>(nc); base += NT) {
        const int i = base + tid;
        const unsigned o = i < static_cast<int>(nc) ? (ckey ? s_ckey[i] : __ldcg(keys + s_cand[i])) : 0u;
        const unsigned gt = i < static_cast<int>(nc) && o > thr, eq = i < static_cast<int>(nc) && o == thr;
        const unsigned packed = (gt << 16) | eq;
        const unsigned incl = block_inclusive_scan(packed, s_warp);
        const unsigned excl = incl - packed;
        const unsigned eq_before = eq_seen + (excl & 0xFFFFu);
        const unsigned at = taken + (excl >> 16) + min(eq_before, need_eq) - min(eq_seen, need_eq);
        if ((gt || (eq && eq_before < need_eq)) && at < static_cast<unsigned>(kTopkTaken)) s_took[at] = s_cand[i];
        if (tid == NT - 1) {
          s_round[0] = incl >> 16;
          s_round[1] = incl & 0xFFFFu;
        }
        __syncthreads();
        const unsigned rg = s_round[0], re = s_round[1];
        taken += rg + min(eq_seen + re, need_eq) - min(eq_seen, need_eq);
        eq_seen += re;
        __syncthreads();
      }
      // merge the two ascending lists
      for (int i = tid; i < static_cast<int>(na); i += NT) {
        const int v = s_above[i];
        const int idx = i + lower_bound_s(s_took, ntake, v);
        sel[idx] = inf.s1 + v;
        if (keep) s_list[idx] = inf.s1 + v;
      }
      for (int j = tid; j < ntake; j += NT) {
        const int v = s_took[j];
        const int idx = j + lower_bound_s(s_above, static_cast<int>(na), v);
        sel[idx] = inf.s1 + v;
        if (keep) s_list[idx] = inf.s1 + v;
      }
    } else {
      // ordered compaction over every key: per round, warp w turns keys
      // [base + 1024 w, base + 1024 (w + 1)) into 32 words (above thr; equal to
      // it), and block scans over the packed popcounts give each word's place
      unsigned gt_seen = 0, eq_seen = 0;
      for (int base = 0; base < mlen; base += 1024 * NWK) {
        const int wb = base + warp * 1024;
        unsigned wgt = 0, weq = 0;
#pragma unroll 4
        for (int j = 0; j < 32; j++) {
          const int x = wb + j * 32 + lane;
          const unsigned o = x < mlen ? __ldcg(keys + x) : 0u;
          const unsigned bg = __ballot_sync(0xffffffffu, x < mlen && o > thr);
          const unsigned be = __ballot_sync(0xffffffffu, x < mlen && o == thr);
          if (lane == j) {
            wgt = bg;
            weq = be;
          }
        }
        const unsigned ng = __popc(wgt), ne = __popc(weq);
        const unsigned incl = block_inclusive_scan((ng << 16) | ne, s_warp);
        const unsigned excl = incl - ((ng << 16) | ne);
        const unsigned gt_before = gt_seen + (excl >> 16), eq_before = eq_seen + (excl & 0xFFFFu);
        const unsigned keepn = need_eq > eq_before ? min(ne, need_eq - eq_before) : 0u;
        unsigned wsel = wgt, e = weq;
        for (unsigned c = 0; c < keepn; c++) {  // the lowest keepn tied positions
          wsel |= e & (0u - e);
          e &= e - 1u;
        }
        unsigned pos = gt_before + min(eq_before, need_eq);
        while (wsel) {
          const int j = inf.s1 + wb + lane * 32 + (__ffs(wsel) - 1);
          sel[pos] = j;
          if (keep) s_list[pos] = j;
          pos++;
          wsel &= wsel - 1u;
        }
        if (tid == NT - 1) {
          s_round[0] = incl & 0xFFFFu;
          s_round[1] = incl >> 16;
        }
        __syncthreads();
        eq_seen += s_round[0];
        gt_seen += s_round[1];
        __syncthreads();
      }
    }
    __syncthreads();  // the list is complete (shared memory, and the global copy for this CTA)
    if (keep) topk = s_list;
  }

  // pilot draws (mode 2), or the whole tail when it is no larger than the pilot (mode 1)
  const int t1 = inf.mode == 2 ? inf.p : (inf.mode == 1 ? inf.ntail : 0);
  const bool whole = inf.mode == 1;
  int* dsel = P.sel + static_cast<size_t>(u) * P.max_ctx + inf.nI;
  // the draw counter names the sequence and KV head in the whole batch (a
  // shard adds its offsets), so a shard draws what the whole batch would
  const unsigned bb = static_cast<unsigned>(P.batch_offset + u / P.Hkv),
                 hh = static_cast<unsigned>(P.head_offset + u % P.Hkv);
  for (int t = tid; t < t1; t += NT) {
    const int rho = whole ? t : lemire(draw_word(P.seed, bb, hh, static_cast<unsigned>(t)), inf.ntail);
    dsel[t] = tail_position(topk, inf.k, inf.s1, rho);
  }
  grid_dependents_launch();
}

// ============================================================ k_draws
// Positions of the sample's entries after the budget: draws t in [p, b), or
// the whole tail when the budget covers it; CTA (0, 0) also writes the sample
// gather's slice prefix (every budget is known by now). Grid (units, splits).
__global__ void __launch_bounds__(128) k_draws(DevParams P) {
  __shared__ int s_topk[kTopkSmem];
  grid_dependency_wait();
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    __shared__ unsigned s_warp[32];
    __shared__ long long s_carry;
    write_slice_prefix<kModeSample>(P, P.pre_samp, s_warp, &s_carry);
    __syncthreads();
  }
  const int u = blockIdx.x;
  const UnitInfo inf = P.info[u];
  int t0 = 0, t1 = 0;
  bool whole = false;
  if (inf.mode == 2) {
    whole = inf.exhausted != 0;
    t0 = whole ? 0 : inf.p;
    t1 = whole ? inf.ntail : inf.bsz;
  }
  const int a = t0 + static_cast<int>(static_cast<long long>(t1 - t0) * blockIdx.y / gridDim.y);
  const int e = t0 + static_cast<int>(static_cast<long long>(t1 - t0) * (blockIdx.y + 1) / gridDim.y);
  if (a < e) write_draw_positions(P, u, inf, whole, a, e, s_topk);
  grid_dependents_launch();
}

// ============================================================ k_budget
// One CTA per unit: the per-head CLT budget from the det gather's records
// (score maxima) and true scores.
constexpr int kBudgetThreads = 512;
template <int D, int G>
__global__ void __launch_bounds__(kBudgetThreads) k_budget(DevParams P) {
  __shared__ float s_mh[G];
  grid_dependency_wait();
  const int u = blockIdx.x;
  const UnitInfo inf = P.info[u];
  const float* ps = P.pscore + static_cast<size_t>(u) * P.max_ctx * G;
  // the scores' first batch is in flight while the maxima are found
  float first[kBudgetBatch][G];
  load_budget_batch<G>(ps, inf.mode == 2 ? inf.nI + inf.p : 0, first);
  if (inf.mode == 2) det_record_max<D, G>(P, u, s_mh);
  unit_budget<G>(P, u, inf, ps, s_mh, first);
  grid_dependents_launch();
}

// ============================================================ k_numstats
// Output guarantee: the numerator part of each query head's budget, from the
// pilot. Grid (units, ceil(G * D / kNumThreads)); thread t of CTA y serves
// head g = (y * kNumThreads + t) / D, dimension e = (y * kNumThreads + t) % D.
// Items are I_f (list order) then the pilot draws (draw order), with their
// true scores s and x = vexp(s - m_h) as in the budget. In double, with each
// product x * v exact (24 x 24 significant bits at most) and every sum in
// item order:
//   A = sum over I_f of x v_e;  T1, T2 = sums over the pilot of y, y * y, y = x v_e;
//   var_e = max(0, (p T2 - T1^2) / (p (p - 1)));  Nv_e = A + N_tail T1 / p.
// One thread per head then sums var_e and Nv_e^2 over e ascending into tr and
// |Nv_hat|^2. The pilot mean's noise has energy R = N_tail^2 tr / p; the lower
// confidence bound L = (|Nv_hat|^2 - R) - z sqrt(4 max(|Nv_hat|^2 - R, 0) R + 2 R^2)
// stands for |Nv|^2, and the kernel writes
//   n_v = (z N_tail / eps)^2 tr / L   (the whole tail when L <= 0 < tr)
// to num_need; k_budget takes max(n_h, n_v). The items' row indices are
// looked up once per block of kNumOffItems items (one parallel pass over
// sel and the page table); the V rows and the true scores of each round of
// items then stream through a kNumStages-deep ring of shared-memory buffers
// by cp.async copies, and x is computed once per (item, head) when a round
// has landed.
constexpr int kNumThreads = 128;
constexpr int kNumBufBytes = 16384;
constexpr int kNumStages = 3;
constexpr int kNumOffItems = 4096;
constexpr size_t kNumSmem = static_cast<size_t>(kNumStages) * kNumBufBytes + kNumOffItems * 4;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kNumThreads) k_numstats(DevParams P) {
  constexpr int HPB = kNumThreads / D;                      // heads per CTA (1 or 2)
  constexpr int ROWB = D * static_cast<int>(sizeof(T));     // bytes per V row
  constexpr int CH = kNumBufBytes / ROWB;                   // items per round
  constexpr int V16 = ROWB / 16;                            // 16-byte pieces per row
  static_assert(kNumOffItems % CH == 0, "rounds must not straddle offset blocks");
  extern __shared__ __align__(16) unsigned char num_smem[];
  unsigned char* s_v = num_smem;                                                    // [stages][16 KB]
  unsigned* s_row = reinterpret_cast<unsigned*>(num_smem + kNumStages * kNumBufBytes);  // [kNumOffItems]
  __shared__ float s_ps[kNumStages][CH * G];  // true scores of a round, [item][head]
  __shared__ double s_x[CH][HPB];
  __shared__ float s_mh[G];
  __shared__ double s_red[2][kNumThreads];
  grid_dependency_wait();
  const int u = blockIdx.x;
  const UnitInfo inf = P.info[u];
  if (inf.mode != 2) {
    grid_dependents_launch();
    return;
  }
  det_record_max<D, G>(P, u, s_mh);
  const int b = u / P.Hkv, h = u % P.Hkv;
  const int tid = threadIdx.x;
  const int g0 = blockIdx.y * HPB;
  const int hh = tid / D, e = tid % D;
  const bool active = g0 + hh < G;
  const int nA = inf.nI + inf.p;
  const int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx;
  const float* ps = P.pscore + static_cast<size_t>(u) * P.max_ctx * G;
  const char* vb = static_cast<const char*>(P.v);
  double A = 0.0, T1 = 0.0, T2 = 0.0;
  for (int s0 = 0; s0 < nA; s0 += kNumOffItems) {
    const int ns = min(kNumOffItems, nA - s0);
    __syncthreads();  // the previous block's rounds are done with s_row and the ring
#pragma unroll 4
    for (int i = tid; i < ns; i += kNumThreads)
      s_row[i] = static_cast<unsigned>(row_off(P, b, h, sel[s0 + i], 1));
    __syncthreads();
    const int rounds = (ns + CH - 1) / CH;
    auto issue = [&](int r) {
      const int c0 = r * CH, cnt = min(CH, ns - c0), buf = r % kNumStages;
      unsigned char* dst = s_v + buf * kNumBufBytes;
      for (int x = tid; x < cnt * V16; x += kNumThreads) {
        const int i = x / V16, k = x % V16;
        const char* src = vb + static_cast<size_t>(s_row[c0 + i]) * ROWB + k * 16;
        if (P.kv_host)  // mapped host memory: a plain load (the round's use waits on a barrier)
          *reinterpret_cast<uint4*>(dst + i * ROWB + k * 16) = ld_gather(src);
        else
          cp_async16(dst + i * ROWB + k * 16, src);
      }
      const float* src = ps + static_cast<size_t>(s0 + c0) * G;
      for (int x = tid; x < cnt * G; x += kNumThreads) cp_async4(&s_ps[buf][x], src + x);
    };
#pragma unroll
    for (int r = 0; r < kNumStages - 1; r++) {
      if (r < rounds) issue(r);
      cp_async_commit();
    }
    for (int r = 0; r < rounds; r++) {
      cp_async_wait<kNumStages - 2>();  // this thread's copies of round r have landed
      __syncthreads();                  // everyone's have, and round r - 1 is consumed
      if (r + kNumStages - 1 < rounds) issue(r + kNumStages - 1);
      cp_async_commit();
      const int c0 = r * CH, cnt = min(CH, ns - c0), buf = r % kNumStages;
      for (int x = tid; x < cnt * HPB; x += kNumThreads) {
        const int i = x / HPB, j = x % HPB;
        const int g = min(g0 + j, G - 1);
        s_x[i][j] = static_cast<double>(vexp(__fsub_rn(s_ps[buf][i * G + g], s_mh[g])));
      }
      __syncthreads();
      if (active) {
        const T* rows = reinterpret_cast<const T*>(s_v + buf * kNumBufBytes);
        const int nIr = inf.nI - (s0 + c0);  // items [0, nIr) of this round are in I_f
        // x * v is exact in double, so A + x * v rounded once (an FMA) is
        // the same as the rounded sum of the exact product
        const int nIc = max(0, min(cnt, nIr));
#pragma unroll 4
        for (int i = 0; i < nIc; i++)
          A = __fma_rn(s_x[i][hh], static_cast<double>(Elem<T>::load(rows, static_cast<size_t>(i) * D + e)), A);
#pragma unroll 4
        for (int i = nIc; i < cnt; i++) {
          const double y = __dmul_rn(s_x[i][hh], static_cast<double>(Elem<T>::load(rows, static_cast<size_t>(i) * D + e)));
          T1 = __dadd_rn(T1, y);
          T2 = __dadd_rn(T2, __dmul_rn(y, y));
        }
      }
    }
    cp_async_wait<0>();
  }
  const double pd = static_cast<double>(inf.p), nt = static_cast<double>(inf.ntail);
  double ve = __ddiv_rn(__dsub_rn(__dmul_rn(pd, T2), __dmul_rn(T1, T1)),
                        __dmul_rn(pd, static_cast<double>(inf.p - 1)));
  if (ve < 0.0) ve = 0.0;
  const double nv = __dadd_rn(A, __ddiv_rn(__dmul_rn(nt, T1), pd));
  s_red[0][tid] = ve;
  s_red[1][tid] = __dmul_rn(nv, nv);
  __syncthreads();
  if (tid < HPB && g0 + tid < G) {
    double tr = 0.0, nsq = 0.0;
    for (int k = 0; k < D; k++) {
      tr = __dadd_rn(tr, s_red[0][tid * D + k]);
      nsq = __dadd_rn(nsq, s_red[1][tid * D + k]);
    }
    // lower confidence bound of |Nv|^2: nsq_u - z * sqrt(4 max(nsq_u, 0) R + 2 R^2)
    const double R = __dmul_rn(__ddiv_rn(__dmul_rn(nt, nt), pd), tr);
    const double nsq_u = __dsub_rn(nsq, R);
    const double se2 = __dadd_rn(__dmul_rn(__dmul_rn(4.0, nsq_u > 0.0 ? nsq_u : 0.0), R),
                                 __dmul_rn(__dmul_rn(2.0, R), R));
    const double lcb = __dsub_rn(nsq_u, __dmul_rn(P.z, __dsqrt_rn(se2)));
    double need;
    if (lcb > 0.0) {
      const double tv = __ddiv_rn(__dmul_rn(P.z, nt), __dmul_rn(static_cast<double>(P.eps), __dsqrt_rn(lcb)));
      need = __dmul_rn(__dmul_rn(tv, tv), tr);
    } else {
      need = tr > 0.0 ? nt : 0.0;
    }
    P.num_need[u * G + g0 + tid] = need >= nt ? inf.ntail : static_cast<int>(ceil(need));
  }
  grid_dependents_launch();
}

// ============================================================ k_combine
// One CTA per (unit, head) of D / 32 to kCombWarps warps: merge the unit's
// records and write the output.
template <int D, int G, int MODE>
__global__ void __launch_bounds__(kCombWarps * 32, 2) k_combine(DevParams P) {
  grid_dependency_wait();
  unit_combine<D, G, MODE>(P, blockIdx.x, blockIdx.y);
  grid_dependents_launch();
}

// ============================================================ k_wait_check
// Exercises the bounded-wait error path: one warp arms an mbarrier for 16
// bytes that no copy ever delivers (no copy is issued, so nothing is in
// flight at exit), waits with a limit of `tries`, and on timeout sets
// VATTN_DEV_TIMEOUT in the error word, exactly as the copy rings do.
__global__ void __launch_bounds__(32) k_wait_check(unsigned* err, int tries) {
  __shared__ __align__(8) uint64_t s_bar;
  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    mbar_init_fence();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_arrive_expect_tx(&s_bar, 16u);
  __syncwarp();
  if (!__all_sync(0xffffffffu, mbar_wait(&s_bar, 0u, tries)) && threadIdx.x == 0) atomicOr(err, kDevTimeout);
}

}  // namespace vattn
