"""Seeded synthetic decode-step inputs.

This module only draws inputs; it holds none of the decode step's arithmetic.
The tests, the benchmark and the oracle all take their inputs from here.

Workloads (long-context decode shapes; the pages evaluate on RULER, LongBench,
Loogle and AIME2024 with Llama/Mistral/DeepSeek checkpoints, none of which is
used here, and these synthetic inputs stand in for them):

  tiny_f32      B1, 4 query = 4 KV heads, d64, N=4096, fp32. q, K, V ~ N(0,1);
                8 planted keys per head at random middle positions,
                k = 4*q/|q| + N(0, 0.1^2).
  gqa_32k       B8, 32 query / 8 KV heads, d128, N=32768, bf16 (Llama-3-8B
                shaped). K, V ~ N(0,1); 1% of positions per KV head set to
                3*qbar/|qbar| + N(0, 0.1^2), qbar the group-mean query.
  sparq_128k    B4, 32/8, d128, N=131072, bf16. k[j,i] = g*exp(0.5*xi_i) with
                g ~ N(0,1) and xi ~ N(0,1) per (sequence, KV head, channel);
                a dim-major copy of K is stored for the r=32 proxy.
  loki_64k      B8, 32/8, d128, N=65536, bf16. k = F @ B_h^T + N(0, 0.1^2),
                F ~ N(0,1)^(N x 32), B_h the orthonormal factor of a Gaussian
                128x32 (per KV head); projected keys bf16(k @ B_h) stored
                alongside.
  paged_sweep   B32, 32/8, d128, N_b ~ U{16384..65536}, page size 16, pages a
                random permutation of the pool; K, V ~ N(0, 0.3^2).

q ~ N(0,1) per query head everywhere. Values are drawn in fp32 and cast.
"""
import dataclasses

import torch

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str              # "f32" | "bf16"
    max_ctx: int
    min_ctx: int            # == max_ctx for fixed-length batches
    page_size: int          # == max_ctx for one contiguous page per sequence
    proxy: str              # "exact" | "sparq" | "loki"
    proxy_rank: int
    sinks: int
    window: int
    topk_abs: int
    topk_num: int
    topk_den: int
    pilot_min: int
    pilot_num: int
    pilot_den: int
    eps: float
    delta: float
    seed: int               # sampler seed
    data_seed: int
    recipe: str
    guarantee: str = "denominator"  # "denominator" | "output": what the budget bounds
    topp_num: int = 0       # topp_den > 0: top-p selection, p = topp_num / topp_den
    topp_den: int = 0

    @property
    def pages_per_seq(self):
        return -(-self.max_ctx // self.page_size)

    @property
    def group(self):
        return self.num_q_heads // self.num_kv_heads

    @property
    def units(self):
        return self.batch * self.num_kv_heads

    def replace(self, **kw):
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 4, 4, 64, "f32", 4096, 4096, 4096, "exact", 0,
                         4, 64, 128, 0, 0, 64, 0, 0, 0.05, 0.05, 0, 1, "planted_q"),
    "gqa_32k": Workload("gqa_32k", 8, 32, 8, 128, "bf16", 32768, 32768, 32768, "exact", 0,
                        128, 128, 0, 2, 100, 64, 1, 100, 0.05, 0.05, 0, 2, "planted_qbar"),
    "sparq_128k": Workload("sparq_128k", 4, 32, 8, 128, "bf16", 131072, 131072, 131072, "sparq", 32,
                           128, 256, 0, 1, 100, 64, 1, 100, 0.05, 0.05, 0, 3, "lognormal_channels"),
    "loki_64k": Workload("loki_64k", 8, 32, 8, 128, "bf16", 65536, 65536, 65536, "loki", 32,
                         64, 128, 0, 2, 100, 64, 1, 100, 0.1, 0.05, 0, 4, "low_rank"),
    "paged_sweep": Workload("paged_sweep", 32, 32, 8, 128, "bf16", 65536, 16384, 16, "exact", 0,
                            128, 128, 0, 1, 100, 64, 1, 100, 0.05, 0.05, 0, 5, "flat"),
}

# the error targets swept on the paged workload
PAGED_EPS_SWEEP = (0.01, 0.05, 0.1, 0.2)


def scaled(w, *, max_ctx, min_ctx=None, batch=None, page_size=None, **kw):
    """Same recipe at a smaller size (a contiguous cache keeps one page per sequence,
    its size max_ctx rounded up to a multiple of 16)."""
    min_ctx = max_ctx if min_ctx is None else min_ctx
    if page_size is None:
        page_size = -(-max_ctx // 16) * 16 if w.page_size >= w.max_ctx else w.page_size
    return w.replace(max_ctx=max_ctx, min_ctx=min_ctx, page_size=page_size,
                     batch=w.batch if batch is None else batch, **kw)


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def make_inputs(w, device="cpu"):
    """Draw one decode step's inputs for workload `w` on `device`.

    Returns a dict: q [B,Hq,d]; k_cache, v_cache [pages][Hkv][page_size][d];
    page_table int32 [B][pages_per_seq] (-1 where unused); seq_lens int32 [B];
    num_pages; and, per proxy, k_t_cache [pages][Hkv][d][page_size] or
    k_proj_cache [pages][Hkv][page_size][rank] with proj_basis fp32 [Hkv][d][rank].
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.data_seed)
    B, Hq, Hkv, d, G = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.group
    dt = _DT[w.dtype]
    ps, pps = w.page_size, w.pages_per_seq

    if w.min_ctx == w.max_ctx:
        seq_lens = torch.full((B,), w.max_ctx, dtype=torch.int32, device=dev)
    else:
        seq_lens = torch.randint(w.min_ctx, w.max_ctx + 1, (B,), generator=g, device=dev,
                                 dtype=torch.int64).to(torch.int32)
    lens = seq_lens.tolist()
    npages = [-(-n // ps) for n in lens]
    total_pages = sum(npages)
    if ps >= w.max_ctx:
        perm = torch.arange(total_pages, device=dev)
    else:
        perm = torch.randperm(total_pages, generator=g, device=dev)
    page_table = torch.full((B, pps), -1, dtype=torch.int32, device=dev)
    starts = [0]
    for n in npages:
        starts.append(starts[-1] + n)
    for b in range(B):
        page_table[b, :npages[b]] = perm[starts[b]:starts[b + 1]].to(torch.int32)

    q32 = _randn((B, Hq, d), g, dev)
    q = q32.to(dt)
    qf = q.float()

    k_cache = torch.empty((total_pages, Hkv, ps, d), dtype=dt, device=dev)
    v_cache = torch.empty((total_pages, Hkv, ps, d), dtype=dt, device=dev)
    out = dict(q=q, k_cache=k_cache, v_cache=v_cache, page_table=page_table,
               seq_lens=seq_lens, num_pages=total_pages)
    rank = w.proxy_rank
    if w.proxy == "sparq":
        out["k_t_cache"] = torch.empty((total_pages, Hkv, d, ps), dtype=dt, device=dev)
    if w.proxy == "loki":
        out["k_proj_cache"] = torch.empty((total_pages, Hkv, ps, rank), dtype=dt, device=dev)
        basis = torch.empty((Hkv, d, rank), dtype=torch.float32, device=dev)
        for h in range(Hkv):
            qmat, _ = torch.linalg.qr(_randn((d, rank), g, dev).cpu())
            basis[h] = qmat.to(dev)
        out["proj_basis"] = basis

    for b in range(B):
        n_b, np_b = lens[b], npages[b]
        rows = np_b * ps                       # logical rows incl. the last page's slack
        if w.recipe == "flat":
            K = 0.3 * _randn((Hkv, rows, d), g, dev)
            V = 0.3 * _randn((Hkv, rows, d), g, dev)
        elif w.recipe == "lognormal_channels":
            xi = _randn((Hkv, 1, d), g, dev)
            K = _randn((Hkv, rows, d), g, dev) * torch.exp(0.5 * xi)
            V = _randn((Hkv, rows, d), g, dev)
        elif w.recipe == "low_rank":
            F = _randn((Hkv, rows, rank), g, dev)
            K = torch.matmul(F, out["proj_basis"].transpose(1, 2)) + 0.1 * _randn((Hkv, rows, d), g, dev)
            V = _randn((Hkv, rows, d), g, dev)
        else:
            K = _randn((Hkv, rows, d), g, dev)
            V = _randn((Hkv, rows, d), g, dev)
            if w.recipe == "planted_q":
                # 8 keys per head aligned with that head's query (one query per KV head)
                lo = min(w.sinks, n_b)
                hi = max(n_b - w.window, lo)
                for h in range(Hkv):
                    if hi - lo <= 0:
                        continue
                    cnt = min(8, hi - lo)
                    pos = lo + torch.randperm(hi - lo, generator=g, device=dev)[:cnt]
                    qh = qf[b, h * G]
                    K[h, pos] = 4.0 * qh / qh.norm() + 0.1 * _randn((cnt, d), g, dev)
            elif w.recipe == "planted_qbar":
                # 1% of positions per KV head aligned with the group-mean query
                cnt = max(1, n_b // 100)
                for h in range(Hkv):
                    pos = torch.randperm(n_b, generator=g, device=dev)[:cnt]
                    qbar = qf[b, h * G:(h + 1) * G].mean(0)
                    K[h, pos] = 3.0 * qbar / qbar.norm() + 0.1 * _randn((cnt, d), g, dev)
        Kc = K.to(dt)
        pages = page_table[b, :np_b].long()
        k_cache[pages] = Kc.view(Hkv, np_b, ps, d).transpose(0, 1)
        v_cache[pages] = V.to(dt).view(Hkv, np_b, ps, d).transpose(0, 1)
        if w.proxy == "sparq":
            out["k_t_cache"][pages] = Kc.view(Hkv, np_b, ps, d).permute(1, 0, 3, 2)
        if w.proxy == "loki":
            kp = torch.matmul(Kc.float(), out["proj_basis"]).to(dt)     # [Hkv, rows, rank]
            out["k_proj_cache"][pages] = kp.view(Hkv, np_b, ps, rank).transpose(0, 1)
        del K, V, Kc
    return out


def bytes_per_elem(w):
    return 4 if w.dtype == "f32" else 2


def describe(w):
    return (f"{w.name}: B{w.batch} Hq{w.num_q_heads}/Hkv{w.num_kv_heads} d{w.head_dim} {w.dtype} "
            f"N={'%d' % w.max_ctx if w.min_ctx == w.max_ctx else '%d..%d' % (w.min_ctx, w.max_ctx)} "
            f"ps{w.page_size} {w.proxy}{'' if w.proxy == 'exact' else ' r%d' % w.proxy_rank} "
            f"s{w.sinks} w{w.window} eps{w.eps} delta{w.delta}"
            + ("" if w.guarantee == "denominator" else f" guarantee={w.guarantee}")
            + ("" if not w.topp_den else f" top-p {w.topp_num}/{w.topp_den}"))


__all__ = ["Workload", "WORKLOADS", "PAGED_EPS_SWEEP", "scaled", "make_inputs", "bytes_per_elem",
           "describe"]
