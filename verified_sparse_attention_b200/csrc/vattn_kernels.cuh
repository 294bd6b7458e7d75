// Kernels of one verified-sparse-attention decode step, in launch order:
//
//   k_prep        per unit: validate, regions, ranking query, proxy query,
//                 zero the radix histograms, write sinks/window indices; one
//                 extra CTA writes the score-pass work prefix over units
//   k_score_rows  exact (q.k) or Loki (projected q . projected k) ranking
//                 scores over the middle region, streamed from HBM; writes
//                 order keys and the first radix digit's histogram
//   k_score_sparq SparQ proxy scores from the dim-major K copy
//   k_sel_hist    radix-select digits 2 and 3 (key bits 20..10, 9..0)
//   k_sel_count   exact threshold; counts above / equal per segment
//   k_sel_write   ordered compaction of the top-k positions (ascending)
//   k_pilot       true scores of I_f and the pilot draws (all query heads)
//   k_budget      per-head CLT budgets from fixed-point statistics
//   k_gather      split-K softmax-and-accumulate over I_f and the sample
//   k_combine     merge splits, reweight the sample by N_tail / b, write out
//
// A unit is one (sequence b, KV head h); u = b * Hkv + h. The method follows
// "vAttention: A New Approach to Sparse Attention with Guaranteed Accuracy",
// section "How vAttention Works" and the paragraph after it.
#pragma once

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
  const long long kb = P.topk_den ? (static_cast<long long>(n) * P.topk_num) / P.topk_den
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

// ============================================================ k_prep
template <typename T, int D, int G>
__global__ void __launch_bounds__(128) k_prep(DevParams P) {
  __shared__ float s_q[D];
  __shared__ float s_abs[D];
  __shared__ unsigned s_warp[32];
  __shared__ unsigned s_tot;
  const int tid = threadIdx.x;
  const int u = blockIdx.x;

  if (u == P.units) {
    // work prefix over units for the persistent score pass
    constexpr int V = Elem<T>::kPer16;
    long long carry = 0;
    for (int base = 0; base < P.units; base += blockDim.x) {
      const int uu = base + tid;
      long long w = 0;
      if (uu < P.units) {
        int n = P.seq_lens[uu / P.Hkv];
        if (n < 0 || n > P.max_ctx) n = 0;
        w = score_work(P, n, V);
      }
      // work per unit <= max_ctx <= 2^24, so a 128-unit chunk sum fits in 32 bits
      const unsigned incl = block_inclusive_scan(static_cast<unsigned>(w), s_warp);
      if (uu < P.units) P.prefix[uu] = carry + (incl - static_cast<unsigned>(w));
      if (tid == blockDim.x - 1) s_tot = incl;
      __syncthreads();
      carry += s_tot;
      __syncthreads();
    }
    if (tid == 0) P.prefix[P.units] = carry;
    return;
  }

  const int b = u / P.Hkv, h = u % P.Hkv;
  int n = P.seq_lens[b];
  const bool bad_len = n < 0 || n > P.max_ctx;
  if (bad_len) n = 0;
  const int npages = (n + P.ps - 1) / P.ps;
  int bad = 0;
  for (int i = tid; i < npages; i += blockDim.x) {
    const int pid = P.page_table[static_cast<size_t>(b) * P.pps + i];
    if (pid < 0 || pid >= P.num_pages) bad = 1;
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
    if (tid < P.rank) {
      float acc = 0.0f;
      for (int i = 0; i < D; i++)
        acc = __fmaf_rn(s_q[i], P.basis[(static_cast<size_t>(h) * D + i) * P.rank + tid], acc);
      P.qsel[static_cast<size_t>(u) * D + tid] = acc;
    }
  }

  unsigned* hist = P.hist + static_cast<size_t>(u) * kHistAll;
  for (int i = tid; i < kHistAll; i += blockDim.x) hist[i] = 0u;
  int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx;
  for (int i = tid; i < r.s1; i += blockDim.x) sel[i] = i;
  for (int i = tid; i < n - r.wst; i += blockDim.x) sel[r.s1 + r.k + i] = r.wst + i;
}

// ============================================================ score pass helpers
// Find the unit whose work range contains item `x` (prefix is non-decreasing).
__device__ __forceinline__ int find_unit(const long long* prefix, int units, long long x) {
  int lo = 0, hi = units;  // largest u with prefix[u] <= x
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= x) lo = mid; else hi = mid;
  }
  return lo;
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
  const bool loki = P.proxy == kProxyLoki;
  const void* cache = loki ? P.kp : P.k;
  const float* qsrc = loki ? P.qsel : P.qbar;

  for (int i = threadIdx.x; i < kHist1; i += blockDim.x) s_hist[i] = 0u;
  __syncthreads();

  const long long total = P.prefix[P.units];
  const long long beg = total * blockIdx.x / gridDim.x;
  const long long end = total * (blockIdx.x + 1) / gridDim.x;
  if (beg >= end) return;
  int u = find_unit(P.prefix, P.units, beg);
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
      flush_hist(s_hist, P.hist + static_cast<size_t>(u) * kHistAll);
    }
    cur = uend;
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

  for (int i = threadIdx.x; i < kHist1; i += blockDim.x) s_hist[i] = 0u;
  __syncthreads();
  const long long total = P.prefix[P.units];
  const long long beg = total * blockIdx.x / gridDim.x;
  const long long end = total * (blockIdx.x + 1) / gridDim.x;
  if (beg >= end) return;
  const int r = P.rank;
  int u = find_unit(P.prefix, P.units, beg);
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
        for (; t + 8 <= r; t += 8) {
          uint4 raw[8];
#pragma unroll
          for (int c = 0; c < 8; c++)
            raw[c] = ld_stream(kt + rowbase + static_cast<size_t>(s_dim[t + c]) * ps + off);
#pragma unroll
          for (int c = 0; c < 8; c++) {
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
      flush_hist(s_hist, P.hist + static_cast<size_t>(u) * kHistAll);
    }
    cur = uend;
  }
}

// ============================================================ radix select
// Digits resolved so far for unit u, recomputed by each CTA from the global
// histograms (cheap: three block scans).
struct SelState {
  int d1, d2, d3, krem;
};

template <int DEPTH>
__device__ __forceinline__ SelState resolve_digits(const DevParams& P, int u, int k) {
  __shared__ int s_digit, s_krem;
  __shared__ unsigned s_warp[32];
  const unsigned* hist = P.hist + static_cast<size_t>(u) * kHistAll;
  SelState st{0, 0, 0, k};
  if (threadIdx.x == 0) { s_digit = 0; s_krem = k; }
  __syncthreads();
  find_digit(hist, kHist1, st.krem, &s_digit, &s_krem, s_warp);
  st.d1 = s_digit;
  st.krem = s_krem;
  __syncthreads();
  if (DEPTH >= 2) {
    find_digit(hist + kHist1, kHist2, st.krem, &s_digit, &s_krem, s_warp);
    st.d2 = s_digit;
    st.krem = s_krem;
    __syncthreads();
  }
  if (DEPTH >= 3) {
    find_digit(hist + kHist1 + kHist2, kHist3, st.krem, &s_digit, &s_krem, s_warp);
    st.d3 = s_digit;
    st.krem = s_krem;
    __syncthreads();
  }
  return st;
}

// Histogram of digit PASS (2 or 3) over keys matching the digits above it.
template <int PASS>
__global__ void __launch_bounds__(256) k_sel_hist(DevParams P) {
  __shared__ unsigned s_h[kHist2];
  const int u = blockIdx.x, seg = blockIdx.y;
  const UnitInfo inf = P.info[u];
  if (inf.k <= 0) return;
  const int pb = inf.s1 + seg * kSeg;
  const int pe = min(inf.wst, pb + kSeg);
  if (pb >= pe) return;
  const SelState st = resolve_digits<PASS - 1>(P, u, inf.k);
  constexpr int NB = PASS == 2 ? kHist2 : kHist3;
  for (int i = threadIdx.x; i < NB; i += blockDim.x) s_h[i] = 0u;
  __syncthreads();
  const unsigned* ordk = P.ordk + static_cast<size_t>(u) * P.max_ctx;
  const unsigned pre = PASS == 2 ? static_cast<unsigned>(st.d1)
                                 : (static_cast<unsigned>(st.d1) << 11 | static_cast<unsigned>(st.d2));
  for (int j = pb + threadIdx.x; j < pe; j += blockDim.x) {
    const unsigned o = ordk[j];
    if (PASS == 2) {
      if ((o >> 21) == pre) atomicAdd(&s_h[(o >> 10) & 2047u], 1u);
    } else {
      if ((o >> 10) == pre) atomicAdd(&s_h[o & 1023u], 1u);
    }
  }
  __syncthreads();
  unsigned* g = P.hist + static_cast<size_t>(u) * kHistAll + (PASS == 2 ? kHist1 : kHist1 + kHist2);
  for (int i = threadIdx.x; i < NB; i += blockDim.x)
    if (s_h[i]) atomicAdd(g + i, s_h[i]);
}

// Threshold key thr (the k-th largest) and need_eq (keys equal to thr to take,
// lowest positions first); counts of keys above / equal to thr per segment.
__global__ void __launch_bounds__(256) k_sel_count(DevParams P) {
  __shared__ unsigned s_warp[32];
  const int u = blockIdx.x, seg = blockIdx.y;
  const UnitInfo inf = P.info[u];
  if (inf.k <= 0) return;
  const int pb = inf.s1 + seg * kSeg;
  const int pe = min(inf.wst, pb + kSeg);
  if (pb >= pe) return;
  const SelState st = resolve_digits<3>(P, u, inf.k);
  const unsigned thr = static_cast<unsigned>(st.d1) << 21 | static_cast<unsigned>(st.d2) << 10 |
                       static_cast<unsigned>(st.d3);
  const unsigned* ordk = P.ordk + static_cast<size_t>(u) * P.max_ctx;
  unsigned gt = 0, eq = 0;
  for (int j = pb + threadIdx.x; j < pe; j += blockDim.x) {
    const unsigned o = ordk[j];
    gt += o > thr;
    eq += o == thr;
  }
  gt = block_sum(gt, s_warp);
  eq = block_sum(eq, s_warp);
  if (threadIdx.x == 0) {
    unsigned* c = P.segcnt + (static_cast<size_t>(u) * P.nseg + seg) * 2;
    c[0] = gt;
    c[1] = eq;
    if (seg == 0) {
      P.info[u].thr = thr;
      P.info[u].need_eq = st.krem;
    }
  }
}

// Ordered compaction: each CTA writes the selected positions of its segment
// at their final ascending rank in sel_idx[s1 ...].
__global__ void __launch_bounds__(256) k_sel_write(DevParams P) {
  __shared__ unsigned s_warp[32];
  __shared__ unsigned s_before[2];
  const int u = blockIdx.x, seg = blockIdx.y;
  const UnitInfo inf = P.info[u];
  if (inf.k <= 0) return;
  const int pb = inf.s1 + seg * kSeg;
  const int pe = min(inf.wst, pb + kSeg);
  if (pb >= pe) return;
  const unsigned thr = inf.thr;
  const unsigned need_eq = static_cast<unsigned>(inf.need_eq);
  if (threadIdx.x < 2) {
    unsigned acc = 0;
    for (int s = 0; s < seg; s++) acc += P.segcnt[(static_cast<size_t>(u) * P.nseg + s) * 2 + threadIdx.x];
    s_before[threadIdx.x] = acc;
  }
  __syncthreads();
  const unsigned gt_before = s_before[0], eq_before = s_before[1];
  const unsigned* ordk = P.ordk + static_cast<size_t>(u) * P.max_ctx;
  constexpr int PER = kSeg / 256;
  const int j0 = pb + threadIdx.x * PER;
  unsigned keys[PER];
  unsigned neq = 0;
#pragma unroll
  for (int i = 0; i < PER; i++) {
    const int j = j0 + i;
    keys[i] = j < pe ? ordk[j] : 0u;
    neq += (j < pe) && keys[i] == thr;
  }
  const unsigned eq_incl = block_inclusive_scan(neq, s_warp);
  unsigned eq_rank = eq_before + eq_incl - neq;
  bool take[PER];
  unsigned ntake = 0;
#pragma unroll
  for (int i = 0; i < PER; i++) {
    const int j = j0 + i;
    const bool valid = j < pe;
    const bool e = valid && keys[i] == thr;
    take[i] = valid && (keys[i] > thr || (e && eq_rank < need_eq));
    eq_rank += e;
    ntake += take[i];
  }
  const unsigned take_incl = block_inclusive_scan(ntake, s_warp);
  unsigned pos = gt_before + min(eq_before, need_eq) + take_incl - ntake;
  int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx + inf.s1;
#pragma unroll
  for (int i = 0; i < PER; i++)
    if (take[i]) sel[pos++] = j0 + i;
}

// ============================================================ tail positions
// Position of the rho-th tail element (0-based, ascending) of M minus top-k:
// s1 + rho + c, with c the number of top-k entries t_i with t_i - s1 - i <= rho.
__device__ __forceinline__ int tail_position(const int* topk, int k, int s1, int rho) {
  int lo = 0, hi = k;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (topk[mid] - s1 - mid <= rho) lo = mid + 1; else hi = mid;
  }
  return s1 + rho + lo;
}

// Stage the sorted top-k list of unit u in shared memory when it fits.
__device__ __forceinline__ const int* stage_topk(const DevParams& P, int u, const UnitInfo& inf,
                                                 int* s_topk) {
  const int* g = P.sel + static_cast<size_t>(u) * P.max_ctx + inf.s1;
  if (inf.k > kTopkSmem) return g;
  for (int i = threadIdx.x; i < inf.k; i += blockDim.x) s_topk[i] = g[i];
  __syncthreads();
  return s_topk;
}

// Position of entry i of unit u's selected list (I_f first, then draws).
__device__ __forceinline__ int item_position(const DevParams& P, int u, const UnitInfo& inf,
                                             const int* topk, int i, bool whole_tail) {
  if (i < inf.nI) return P.sel[static_cast<size_t>(u) * P.max_ctx + i];
  const int t = i - inf.nI;
  int rho;
  if (whole_tail) {
    rho = t;
  } else {
    const unsigned w = draw_word(P.seed, static_cast<unsigned>(u / P.Hkv),
                                 static_cast<unsigned>(u % P.Hkv), static_cast<unsigned>(t));
    rho = lemire(w, inf.ntail);
  }
  return tail_position(topk, inf.k, inf.s1, rho);
}

// ============================================================ k_pilot
// True scores s = fl(dot(q_g, k_j) * scale) of every query head of the group,
// for I_f and the p pilot draws, into pscore[u][i][g].
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) k_pilot(DevParams P) {
  constexpr int E = Elem<T>::kPer16;
  constexpr int L = D / E;
  constexpr int RPW = 32 / L;
  __shared__ int s_topk[kTopkSmem];
  const int u = blockIdx.x, a = blockIdx.y;
  const UnitInfo inf = P.info[u];
  if (inf.mode != 2) return;
  const int nA = inf.nI + inf.p;
  const int ib = static_cast<int>(static_cast<long long>(nA) * a / P.SA);
  const int ie = static_cast<int>(static_cast<long long>(nA) * (a + 1) / P.SA);
  if (ib >= ie) return;
  const int* topk = stage_topk(P, u, inf, s_topk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int grp = lane / L, li = lane % L;
  const int b = u / P.Hkv, h = u % P.Hkv;
  float q[G][E];
#pragma unroll
  for (int g = 0; g < G; g++)
#pragma unroll
    for (int e = 0; e < E; e++)
      q[g][e] = Elem<T>::load(P.q, (static_cast<size_t>(b) * P.Hq + h * G + g) * D + li * E + e);
  const T* kc = static_cast<const T*>(P.k);
  float* ps = P.pscore + static_cast<size_t>(u) * P.max_ctx * G;
  constexpr int UU = 2;
  // warp-uniform trip count: every lane runs the shuffles of group_allreduce
  for (int wb = ib + warp * RPW * UU; wb < ie; wb += nwarps * RPW * UU) {
    uint4 raw[UU];
#pragma unroll
    for (int k = 0; k < UU; k++) {
      const int i = wb + k * RPW + grp;
      if (i < ie) {
        const int j = item_position(P, u, inf, topk, i, false);
        raw[k] = ld_gather(kc + row_off(P, b, h, j, D) + li * E);
      } else {
        raw[k] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int k = 0; k < UU; k++) {
      const int i = wb + k * RPW + grp;
#pragma unroll
      for (int g = 0; g < G; g++) {
        const float s = __fmul_rn(group_allreduce<L>(chunk_dot<T>(q[g], raw[k])), P.scale);
        if (li == 0 && i < ie) ps[static_cast<size_t>(i) * G + g] = s;
      }
    }
  }
}

// ============================================================ k_budget
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

// Per query head: m = max score over I_f and the pilot; x = vexp(s - m);
// xq = round(x * 2^32); S_f = sum over I_f, S1 and S2 = sums of xq and xq^2
// over the pilot (integers, so the reduction order does not matter);
// n_h = (z * N_tail * sigma / (eps * D))^2 with sigma^2 = (p S2 - S1^2) /
// (p (p - 1)) and D = S_f + N_tail * S1 / p, evaluated in double in a fixed
// operation order. b = max(p, max_h n_h); b >= N_tail takes the whole tail.
template <int G>
__global__ void __launch_bounds__(256) k_budget(DevParams P) {
  __shared__ float s_m[8];
  __shared__ unsigned long long s_a[8], s_b[8];
  __shared__ U128 s_c[8];
  __shared__ int s_need[G];
  const int u = blockIdx.x;
  const int b = u / P.Hkv, h = u % P.Hkv;
  UnitInfo inf = P.info[u];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  if (inf.mode != 2) {
    if (tid == 0) {
      const int bsz = inf.mode == 1 ? inf.ntail : 0;
      P.info[u].bsz = bsz;
      P.info[u].exhausted = inf.mode == 1;
      P.info[u].nitems = inf.nI + bsz;
      P.budgets[u] = bsz;
      P.sel_count[u] = inf.nI + bsz;
    }
    if (tid < G) P.head_need[static_cast<size_t>(b) * P.Hq + h * G + tid] = inf.mode == 1 ? inf.ntail : 0;
    return;
  }
  const int nA = inf.nI + inf.p;
  const float* ps = P.pscore + static_cast<size_t>(u) * P.max_ctx * G;
  for (int g = 0; g < G; g++) {
    float m = -INFINITY;
    for (int i = tid; i < nA; i += blockDim.x) m = fmaxf(m, ps[static_cast<size_t>(i) * G + g]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_m[warp] = m;
    __syncthreads();
    m = s_m[0];
    for (int w = 1; w < nw; w++) m = fmaxf(m, s_m[w]);
    unsigned long long sf = 0, s1 = 0;
    U128 s2{0ull, 0ull};
    for (int i = tid; i < nA; i += blockDim.x) {
      const float x = vexp(__fsub_rn(ps[static_cast<size_t>(i) * G + g], m));
      const unsigned long long xq = __float2ull_rn(__fmul_rn(x, 4294967296.0f));
      if (i < inf.nI) {
        sf += xq;
      } else {
        s1 += xq;
        s2 = u128_add(s2, U128{xq * xq, __umul64hi(xq, xq)});
      }
    }
    sf = warp_sum_u64(sf);
    s1 = warp_sum_u64(s1);
    s2 = warp_sum_u128(s2);
    __syncthreads();
    if (lane == 0) {
      s_a[warp] = sf;
      s_b[warp] = s1;
      s_c[warp] = s2;
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long Sf = 0, S1 = 0;
      U128 S2{0ull, 0ull};
      for (int w = 0; w < nw; w++) {
        Sf += s_a[w];
        S1 += s_b[w];
        S2 = u128_add(S2, s_c[w]);
      }
      const unsigned long long p = static_cast<unsigned long long>(inf.p);
      // V = p*S2 - S1^2 (exact, >= 0)
      U128 pS2;
      pS2.lo = p * S2.lo;
      pS2.hi = __umul64hi(p, S2.lo) + p * S2.hi;
      const unsigned long long sq_lo = S1 * S1, sq_hi = __umul64hi(S1, S1);
      U128 V;
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
      s_need[g] = need >= nt ? inf.ntail : static_cast<int>(ceil(need));
    }
    __syncthreads();
  }
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
  if (tid < G) P.head_need[static_cast<size_t>(b) * P.Hq + h * G + tid] = s_need[tid];
}

// ============================================================ k_gather
// Split-K softmax-and-accumulate over a contiguous slice [ib, ie) of unit u's
// selected list (all positions, for dense). Entries below nDet carry weight 1
// (I_f, or everything when the tail is taken whole); the rest are sample
// draws. Each part keeps its own softmax state per query head: running max m,
// exp sum l and exp-weighted value sum acc. The slice's two states go to
// partial slot [u][blockIdx.y] as (m_f, l_f, m_s, l_s, acc_f[D], acc_s[D]).
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) k_gather(DevParams P) {
  constexpr int E = Elem<T>::kPer16;
  constexpr int L = D / E;
  constexpr int RPW = 32 / L;
  constexpr int NGRP = 8 * RPW;  // lane groups per CTA (8 warps)
  constexpr int PW = 4 + 2 * D;  // floats per head in a partial
  constexpr int UU = 2;          // rows in flight per lane group
  __shared__ int s_topk[kTopkSmem];
  __shared__ float s_stat[NGRP][G][2];
  __shared__ float s_acc[G][D];

  const int u = blockIdx.x, a = blockIdx.y;
  const UnitInfo inf = P.info[u];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / L, li = lane % L;
  const int gid = warp * RPW + grp;
  const int b = u / P.Hkv, h = u % P.Hkv;

  const int n_items = P.dense ? inf.n : inf.nitems;
  const bool whole_tail = inf.exhausted != 0;
  const int n_det = (P.dense || whole_tail) ? n_items : inf.nI;
  const int ib = static_cast<int>(static_cast<long long>(n_items) * a / P.SB);
  const int ie = static_cast<int>(static_cast<long long>(n_items) * (a + 1) / P.SB);
  const int* topk = s_topk;
  if (!P.dense && ie > inf.nI && ib < ie) topk = stage_topk(P, u, inf, s_topk);

  float q[G][E];
#pragma unroll
  for (int g = 0; g < G; g++)
#pragma unroll
    for (int e = 0; e < E; e++)
      q[g][e] = Elem<T>::load(P.q, (static_cast<size_t>(b) * P.Hq + h * G + g) * D + li * E + e);

  const T* kc = static_cast<const T*>(P.k);
  const T* vc = static_cast<const T*>(P.v);
  int* sel = P.sel + static_cast<size_t>(u) * P.max_ctx;
  float* part = P.partial + (static_cast<size_t>(u) * kSbMax + a) * G * PW;

#pragma unroll 1
  for (int half = 0; half < 2; half++) {
    const int rb = half == 0 ? ib : max(ib, n_det);
    const int re = half == 0 ? min(ie, n_det) : ie;
    float m[G], l[G], acc[G][E];
#pragma unroll
    for (int g = 0; g < G; g++) {
      m[g] = -INFINITY;
      l[g] = 0.0f;
#pragma unroll
      for (int e = 0; e < E; e++) acc[g][e] = 0.0f;
    }
    // warp-uniform trip count: every lane runs the shuffles of group_allreduce
    for (int wb = rb + warp * RPW * UU; wb < re; wb += NGRP * UU) {
      uint4 kr[UU], vr[UU];
      bool ok[UU];
#pragma unroll
      for (int k = 0; k < UU; k++) {
        const int i = wb + k * RPW + grp;
        ok[k] = i < re;
        if (ok[k]) {
          int j = i;
          if (!P.dense) {
            j = item_position(P, u, inf, topk, i, whole_tail);
            if (i >= inf.nI && li == 0) sel[i] = j;
          }
          const size_t off = row_off(P, b, h, j, D) + li * E;
          kr[k] = ld_gather(kc + off);
          vr[k] = ld_gather(vc + off);
        } else {
          kr[k] = vr[k] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      float s[UU][G];
#pragma unroll
      for (int k = 0; k < UU; k++)
#pragma unroll
        for (int g = 0; g < G; g++)
          s[k][g] = __fmul_rn(group_allreduce<L>(chunk_dot<T>(q[g], kr[k])), P.scale);
#pragma unroll
      for (int g = 0; g < G; g++) {
        float mx = m[g];
#pragma unroll
        for (int k = 0; k < UU; k++)
          if (ok[k]) mx = fmaxf(mx, s[k][g]);
        if (mx > m[g]) {
          const float c = __expf(m[g] - mx);  // 0 while m = -inf
          l[g] *= c;
#pragma unroll
          for (int e = 0; e < E; e++) acc[g][e] *= c;
          m[g] = mx;
        }
      }
#pragma unroll
      for (int k = 0; k < UU; k++) {
        if (!ok[k]) continue;
        float x[E];
        Elem<T>::unpack(vr[k], x);
#pragma unroll
        for (int g = 0; g < G; g++) {
          const float e = __expf(s[k][g] - m[g]);
          l[g] += e;
#pragma unroll
          for (int t = 0; t < E; t++) acc[g][t] = fmaf(e, x[t], acc[g][t]);
        }
      }
    }

    // ---- merge the CTA's lane groups into one state for this part
    __syncthreads();
    if (li == 0) {
#pragma unroll
      for (int g = 0; g < G; g++) {
        s_stat[gid][g][0] = m[g];
        s_stat[gid][g][1] = l[g];
      }
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; g++) {
      float mm = -INFINITY;
      for (int x = 0; x < NGRP; x++) mm = fmaxf(mm, s_stat[x][g][0]);
      const float c = (m[g] == -INFINITY) ? 0.0f : __expf(m[g] - mm);
#pragma unroll
      for (int e = 0; e < E; e++) {
        float v = acc[g][e] * c;
#pragma unroll
        for (int o = L; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        acc[g][e] = v;
      }
      if (threadIdx.x == 0) {
        float Lsum = 0.0f;
        for (int x = 0; x < NGRP; x++) {
          const float mx = s_stat[x][g][0];
          Lsum += (mx == -INFINITY) ? 0.0f : s_stat[x][g][1] * __expf(mx - mm);
        }
        part[g * PW + 2 * half] = mm;
        part[g * PW + 2 * half + 1] = Lsum;
      }
    }
    // warps add their sums into s_acc one after another (fixed order)
    for (int w = 0; w < 8; w++) {
      if (warp == w && grp == 0) {
#pragma unroll
        for (int g = 0; g < G; g++)
#pragma unroll
          for (int e = 0; e < E; e++) {
            float& dst = s_acc[g][li * E + e];
            dst = (w == 0) ? acc[g][e] : dst + acc[g][e];
          }
      }
      __syncthreads();
    }
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x)
      part[(idx / D) * PW + 4 + half * D + idx % D] = s_acc[idx / D][idx % D];
  }
}

// ============================================================ k_combine
// Per query head: merge the splits of each part to a common max, then
// out = (A_f + w A_s) / (L_f + w L_s) with w = N_tail / b for a sampled tail
// and 1 otherwise.
template <int D, int G>
__global__ void __launch_bounds__(1024) k_combine(DevParams P) {
  constexpr int PW = 4 + 2 * D;
  const int u = blockIdx.x;
  const int b = u / P.Hkv, h = u % P.Hkv;
  const int g = threadIdx.x / D, e = threadIdx.x % D;
  if (g >= G) return;
  const UnitInfo inf = P.info[u];
  float* out = P.out + (static_cast<size_t>(b) * P.Hq + h * G + g) * D + e;
  if (inf.n <= 0) {
    *out = 0.0f;
    return;
  }
  const float* part = P.partial + static_cast<size_t>(u) * kSbMax * G * PW + g * PW;
  float Mh[2] = {-INFINITY, -INFINITY};
  for (int a = 0; a < P.SB; a++)
    for (int f = 0; f < 2; f++) Mh[f] = fmaxf(Mh[f], part[static_cast<size_t>(a) * G * PW + 2 * f]);
  float Lh[2] = {0.f, 0.f}, Ah[2] = {0.f, 0.f};
  for (int a = 0; a < P.SB; a++) {
    const float* pa = part + static_cast<size_t>(a) * G * PW;
    for (int f = 0; f < 2; f++) {
      const float mx = pa[2 * f];
      const float c = (mx == -INFINITY) ? 0.0f : __expf(mx - Mh[f]);
      Lh[f] += pa[2 * f + 1] * c;
      Ah[f] += pa[4 + f * D + e] * c;
    }
  }
  const float M = fmaxf(Mh[0], Mh[1]);
  const float cf = (Mh[0] == -INFINITY) ? 0.0f : __expf(Mh[0] - M);
  const float cs = (Mh[1] == -INFINITY) ? 0.0f : __expf(Mh[1] - M);
  float w = 1.0f;
  if (!P.dense && inf.mode == 2 && !inf.exhausted)
    w = static_cast<float>(static_cast<double>(inf.ntail) / static_cast<double>(inf.bsz));
  const float num = Ah[0] * cf + w * (Ah[1] * cs);
  const float den = Lh[0] * cf + w * (Lh[1] * cs);
  *out = num / den;
}

}  // namespace vattn
