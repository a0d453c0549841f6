"""Seeded synthetic workloads for decode attention over a cross-layer-compressed KV cache.

This module only draws random tensors and shapes them into the layouts the library
consumes.  It holds none of the method's arithmetic (no scoring, selection,
reconstruction or attention): both the CUDA path and the CPU oracle take its output
as input.

Workloads (shapes and value recipes follow the cross-layer KV pages):

* xKV factors, per window of W layers (xKV, section 2.2 "Cross-Layer Factorization"):
  a shared token basis A (L x r) per sequence, kept separately for keys (r_K) and
  values (r_V), built as Q * diag(s) with Q the orthonormal factor of a Gaussian
  L x r matrix and s_i = exp(-i / tau); and per-layer reconstruction matrices
  B_l (r x d_kv) with entries ~ N(0, 1/r) (variance 1/r).
* Queries ~ N(0, 1/sqrt(hd)) (variance 1/sqrt(hd)).
* "Needle" chunks (Llama-3.1-8B 32K workload): per sequence, a few chunk indices
  outside the sink and recent chunks; query head j of a KV group g (j = 0..G-1 within
  the group) gets lambda * u_n added for needle n = j mod n_needles, u_n the unit
  direction of needle n's mean key (mean of the chunk's A rows times B_l's group-g
  columns), lambda = 4 * hd^(1/4).  One needle per head keeps the needles from
  interfering; the group max still reaches each of them.
* R-CLA leader caches (Stochastic KV Routing page, inference sharing strategy S):
  K, V ~ N(0, 1); 1% of token positions per sequence (shared by leaders and heads)
  have their V row multiplied by 20 (a large value range, as on the VASE page).

Layouts (row-major, last index fastest):
  Ak  [n_win][B][L][r_K]        Av  [n_win][B][L][r_V]
  Bkt [N][B][d_kv][r_K]         Bvt [N][B][d_kv][r_V]   (B_l stored column-major)
  q   [n_q][N][B][Hq][hd]       (n_q = query pool size, step s uses slot s % n_q)
  K_lead, V_lead [n_lead][B][Hkv][L_max][hd]
  k_new, v_new   [n_q][n_lead][B][Hkv][hd]
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "TINY_SR_F32", "LLAMA8B_SR_32K", "QWEN3_8B_RCLA_32K",
    "LLAMA8B_DENSE_128K", "QWEN14B_SR_16K", "reduced", "leader_set",
    "np_basis", "np_recon_t", "np_queries", "np_needle_chunks", "np_plant_needles",
    "np_xkv_layer_inputs", "np_rcla_inputs", "to_storage",
    "torch_xkv_cache", "torch_xkv_layer", "torch_queries", "torch_layer_queries",
    "torch_rcla_cache",
]


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str            # "sr" (selective), "dense", "rcla"
    batch: int
    n_layers: int
    window: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ctx_len: int
    rank_k: int = 0
    rank_v: int = 0
    chunk: int = 8
    top_k: int = 0
    n_sink: int = 0
    n_recent: int = 0
    dtype: str = "bf16"  # "f32" or "bf16"
    steps: int = 1
    tau: float = 16.0
    n_needles: int = 0
    leader_stride: int = 0
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    extra_rows: int = 0  # R-CLA: cache capacity beyond ctx_len (one row per decode step)

    @property
    def d_kv(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_chunks(self) -> int:
        return self.ctx_len // self.chunk

    @property
    def n_windows(self) -> int:
        return -(-self.n_layers // max(self.window, 1))

    @property
    def n_sel(self) -> int:
        """Chunks attended per (sequence, KV head): top-k plus the forced chunks."""
        forced = forced_chunks(self.n_chunks, self.n_sink, self.n_recent)
        cand = self.n_chunks - len(forced)
        return min(self.top_k, cand) + len(forced)

    @property
    def L_max(self) -> int:
        return self.ctx_len + self.extra_rows

    def q_pool(self) -> int:
        return max(1, min(self.steps, 16))


def forced_chunks(n_chunks: int, n_sink: int, n_recent: int) -> list[int]:
    """Sink chunks {0..n_sink-1} and recent chunks {nC-n_recent..nC-1}, deduplicated."""
    f = set(range(min(n_sink, n_chunks)))
    f |= set(range(max(0, n_chunks - n_recent), n_chunks))
    return sorted(f)


def leader_set(w: Workload) -> list[int]:
    return list(range(0, w.n_layers, w.leader_stride))


# The five workloads: tiny fp32 parity case; Llama-3.1-8B-shaped selective decode at
# 32K; Qwen3-8B-shaped R-CLA sharing at 32K; Llama-3.1-8B-shaped dense reconstruction
# at 128K; Qwen2.5-14B-shaped selective decode at 16K with batch 64.
TINY_SR_F32 = Workload("tiny_sr_f32", "sr", batch=1, n_layers=2, window=2, n_q_heads=4,
                       n_kv_heads=2, head_dim=64, ctx_len=1024, rank_k=64, rank_v=64,
                       chunk=8, top_k=16, n_sink=1, n_recent=1, dtype="f32", steps=1,
                       tau=16.0)
LLAMA8B_SR_32K = Workload("llama8b_sr_32k", "sr", batch=8, n_layers=32, window=4,
                          n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=32768,
                          rank_k=512, rank_v=768, chunk=8, top_k=256, n_sink=1, n_recent=4,
                          dtype="bf16", steps=64, tau=128.0, n_needles=4)
QWEN3_8B_RCLA_32K = Workload("qwen3_8b_rcla_32k", "rcla", batch=16, n_layers=36, window=1,
                             n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=32768,
                             dtype="bf16", steps=64, leader_stride=4, outlier_frac=0.01,
                             outlier_scale=20.0, extra_rows=64)
LLAMA8B_DENSE_128K = Workload("llama8b_dense_128k", "dense", batch=1, n_layers=32, window=4,
                              n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=131072,
                              rank_k=512, rank_v=768, chunk=8, dtype="bf16", steps=32,
                              tau=16.0)
QWEN14B_SR_16K = Workload("qwen14b_sr_16k", "sr", batch=64, n_layers=48, window=4,
                          n_q_heads=40, n_kv_heads=8, head_dim=128, ctx_len=16384,
                          rank_k=512, rank_v=768, chunk=8, top_k=128, n_sink=1, n_recent=4,
                          dtype="bf16", steps=128, tau=16.0)

WORKLOADS = {w.name: w for w in (TINY_SR_F32, LLAMA8B_SR_32K, QWEN3_8B_RCLA_32K,
                                 LLAMA8B_DENSE_128K, QWEN14B_SR_16K)}


def reduced(w: Workload, **kw) -> Workload:
    """Same recipe at smaller sizes (defaults: batch 2, 2048 tokens, one window)."""
    kw.setdefault("batch", 2)
    kw.setdefault("ctx_len", 2048)
    if w.mode == "rcla":
        kw.setdefault("n_layers", 8)
        kw.setdefault("extra_rows", 4)
    else:
        kw.setdefault("n_layers", w.window)
    kw.setdefault("steps", 1)
    kw.setdefault("name", w.name + "_reduced")
    return dataclasses.replace(w, **kw)


# ----------------------------------------------------------------------------------
# numpy generators (CPU, fp64 before the cast to the storage dtype): small workloads
# ----------------------------------------------------------------------------------
_TAGS = {"Ak": 1, "Av": 2, "Bk": 3, "Bv": 4, "q": 5, "needle": 6, "K": 7, "V": 8,
         "knew": 9, "vnew": 10, "outlier": 11, "clfU": 12, "clfV": 13, "omega": 14}


def _rng(seed: int, tag: str, *idx: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAGS[tag], *idx])))


def np_basis(w: Workload, seed: int, seq: int, win: int, which: str) -> np.ndarray:
    """A (L x r), fp64: orthonormal factor of a Gaussian matrix times diag(exp(-i/tau))."""
    r = w.rank_k if which == "k" else w.rank_v
    g = _rng(seed, "Ak" if which == "k" else "Av", seq, win)
    q, _ = np.linalg.qr(g.standard_normal((w.ctx_len, r)))
    s = np.exp(-np.arange(r) / w.tau)
    return q * s[None, :]


def np_recon_t(w: Workload, seed: int, seq: int, layer: int, which: str) -> np.ndarray:
    """B_l transposed (d_kv x r), fp64, entries ~ N(0, 1/r)."""
    r = w.rank_k if which == "k" else w.rank_v
    g = _rng(seed, "Bk" if which == "k" else "Bv", seq, layer)
    return g.standard_normal((w.d_kv, r)) / math.sqrt(r)


def np_queries(w: Workload, seed: int, step: int, layer: int) -> np.ndarray:
    """q [B][Hq][hd], fp64, ~ N(0, 1/sqrt(hd))."""
    g = _rng(seed, "q", step, layer)
    return g.standard_normal((w.batch, w.n_q_heads, w.head_dim)) * w.head_dim ** -0.25


def np_needle_chunks(w: Workload, seed: int, seq: int) -> np.ndarray:
    forced = set(forced_chunks(w.n_chunks, w.n_sink, w.n_recent))
    pool = np.array([c for c in range(w.n_chunks) if c not in forced])
    g = _rng(seed, "needle", seq)
    return np.sort(g.choice(pool, size=w.n_needles, replace=False))


def np_plant_needles(w: Workload, q: np.ndarray, Ak_seq: np.ndarray, Bkt_seq: np.ndarray,
                     needles: np.ndarray, seq: int) -> None:
    """Add lambda * u_(j mod n) to head j of each KV group (in place, one sequence)."""
    lam = 4.0 * w.head_dim ** 0.25
    C, hd, G = w.chunk, w.head_dim, w.group
    for g in range(w.n_kv_heads):
        Bg = Bkt_seq[g * hd:(g + 1) * hd, :]               # hd x r
        u = []
        for n in needles:
            abar = Ak_seq[n * C:(n + 1) * C, :].mean(axis=0)
            d = Bg @ abar
            u.append(d / np.linalg.norm(d))
        for j in range(G):
            q[seq, g * G + j, :] += lam * u[j % len(u)]


def window_spectrum(n_modes: int, rank: int, tau: float, gap: float) -> np.ndarray:
    """Singular values of a synthetic window concatenation: exp(-i/tau), times `gap`
    from index `rank` on (gap < 1 puts a drop right after the kept rank)."""
    i = np.arange(n_modes, dtype=np.float64)
    s = np.exp(-i / tau)
    s[rank:] *= gap
    return s


def np_window_caches(W: int, B: int, L: int, d_kv: int, n_modes: int, rank: int,
                     tau: float, gap: float, seed: int):
    """Caches of a window of W layers whose layers share one token subspace (the xKV
    page's observation, section 2.1), with a known spectrum: per sequence the
    concatenation [X_0 | ... | X_{W-1}] is exactly U diag(s) V^T, U (L x m) and V
    (W·d_kv x m) with orthonormal columns (QR of Gaussian matrices), s from
    window_spectrum, m = min(n_modes, L, W·d_kv); X_l = U diag(s) V_l^T with V_l the
    l-th block of d_kv rows of V.  Returns (X [W][B][L][d_kv] fp64, s [m])."""
    n = W * d_kv
    m = min(n_modes, L, n)
    s = window_spectrum(m, rank, tau, gap)
    X = np.empty((W, B, L, d_kv))
    for b in range(B):
        U, _ = np.linalg.qr(_rng(seed, "clfU", b).standard_normal((L, m)))
        V, _ = np.linalg.qr(_rng(seed, "clfV", b).standard_normal((n, m)))
        US = U * s[None, :]
        for l in range(W):
            X[l, b] = US @ V[l * d_kv:(l + 1) * d_kv].T
    return X, s


def np_test_matrix(n: int, rank: int, seed: int) -> np.ndarray:
    """The Gaussian test matrix of the randomized range finder, n x r, fp32."""
    return _rng(seed, "omega", n, rank).standard_normal((n, rank)).astype(np.float32)


def to_storage(x: np.ndarray, dtype: str):
    """fp64 numpy -> torch CPU tensor in the storage dtype (deterministic cast)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    return t.to(torch.float32).contiguous() if dtype == "f32" else t.to(torch.bfloat16).contiguous()


def np_xkv_layer_inputs(w: Workload, seed: int, layer: int, step: int = 0,
                        needles_from: "tuple | None" = None) -> dict:
    """Everything one layer of an xKV step needs, as torch CPU tensors in storage dtype.

    Returns Ak [B][L][rk], Av [B][L][rv], Bkt [B][d_kv][rk], Bvt [B][d_kv][rv],
    q [B][Hq][hd], and the needle chunk indices per sequence (if any).
    """
    win = layer // w.window
    Ak = np.stack([np_basis(w, seed, b, win, "k") for b in range(w.batch)])
    Av = np.stack([np_basis(w, seed, b, win, "v") for b in range(w.batch)])
    Bkt = np.stack([np_recon_t(w, seed, b, layer, "k") for b in range(w.batch)])
    Bvt = np.stack([np_recon_t(w, seed, b, layer, "v") for b in range(w.batch)])
    q = np_queries(w, seed, step, layer)
    needles = []
    for b in range(w.batch):
        if w.n_needles:
            nd = np_needle_chunks(w, seed, b)
            np_plant_needles(w, q, Ak[b], Bkt[b], nd, b)
            needles.append(nd)
    out = {k: to_storage(v, w.dtype) for k, v in
           dict(Ak=Ak, Av=Av, Bkt=Bkt, Bvt=Bvt, q=q).items()}
    out["needles"] = needles
    return out


def np_rcla_inputs(w: Workload, seed: int, len_rows: int, step: int = 0) -> dict:
    """Leader caches and one step's queries / new rows, torch CPU tensors (storage dtype).

    K_lead, V_lead [n_lead][B][Hkv][L_max][hd] hold len_rows valid rows (the rest zero);
    q [N][B][Hq][hd]; k_new, v_new [n_lead][B][Hkv][hd].
    """
    S = leader_set(w)
    nl, B, H, Lm, hd = len(S), w.batch, w.n_kv_heads, w.L_max, w.head_dim
    K = np.zeros((nl, B, H, Lm, hd))
    V = np.zeros((nl, B, H, Lm, hd))
    for s in range(nl):
        for b in range(B):
            K[s, b, :, :len_rows] = _rng(seed, "K", s, b).standard_normal((H, len_rows, hd))
            V[s, b, :, :len_rows] = _rng(seed, "V", s, b).standard_normal((H, len_rows, hd))
    for b in range(B):
        n_out = int(round(w.outlier_frac * len_rows))
        if n_out:
            pos = _rng(seed, "outlier", b).choice(len_rows, size=n_out, replace=False)
            V[:, b, :, pos, :] *= w.outlier_scale
    q = np.stack([np_queries(w, seed, step, l) for l in range(w.n_layers)])
    kn = _rng(seed, "knew", step).standard_normal((nl, B, H, hd))
    vn = _rng(seed, "vnew", step).standard_normal((nl, B, H, hd))
    return {k: to_storage(v, w.dtype) for k, v in
            dict(K_lead=K, V_lead=V, q=q, k_new=kn, v_new=vn).items()}


# ----------------------------------------------------------------------------------
# torch generators (on a device, fp32 before the cast): full-size workloads
# ----------------------------------------------------------------------------------
def _tgen(seed: int, tag: str, *idx: int, device="cuda"):
    import torch
    ss = np.random.SeedSequence([seed, _TAGS[tag], *idx])
    g = torch.Generator(device=device)
    g.manual_seed(int(ss.generate_state(1, dtype=np.uint64)[0] & ((1 << 63) - 1)))
    return g


def _tdtype(dtype: str):
    import torch
    return torch.float32 if dtype == "f32" else torch.bfloat16


def _t_basis(w: Workload, seed: int, seq: int, win: int, which: str, device):
    import torch
    r = w.rank_k if which == "k" else w.rank_v
    g = _tgen(seed, "Ak" if which == "k" else "Av", seq, win, device=device)
    x = torch.randn((w.ctx_len, r), generator=g, device=device, dtype=torch.float32)
    qf, _ = torch.linalg.qr(x)
    s = torch.exp(-torch.arange(r, device=device, dtype=torch.float32) / w.tau)
    return (qf * s[None, :]).to(_tdtype(w.dtype))


def _t_recon_t(w: Workload, seed: int, seq: int, layer: int, which: str, device):
    import torch
    r = w.rank_k if which == "k" else w.rank_v
    g = _tgen(seed, "Bk" if which == "k" else "Bv", seq, layer, device=device)
    return (torch.randn((w.d_kv, r), generator=g, device=device) / math.sqrt(r)).to(
        _tdtype(w.dtype))


def torch_xkv_cache(w: Workload, seed: int, device="cuda") -> dict:
    """Full xKV cache on a device: Ak, Av [n_win][B][L][r], Bkt, Bvt [N][B][d_kv][r]."""
    import torch
    dt = _tdtype(w.dtype)
    Ak = torch.empty((w.n_windows, w.batch, w.ctx_len, w.rank_k), dtype=dt, device=device)
    Av = torch.empty((w.n_windows, w.batch, w.ctx_len, w.rank_v), dtype=dt, device=device)
    for win in range(w.n_windows):
        for b in range(w.batch):
            Ak[win, b].copy_(_t_basis(w, seed, b, win, "k", device))
            Av[win, b].copy_(_t_basis(w, seed, b, win, "v", device))
    Bkt = torch.empty((w.n_layers, w.batch, w.d_kv, w.rank_k), dtype=dt, device=device)
    Bvt = torch.empty((w.n_layers, w.batch, w.d_kv, w.rank_v), dtype=dt, device=device)
    for l in range(w.n_layers):
        for b in range(w.batch):
            Bkt[l, b].copy_(_t_recon_t(w, seed, b, l, "k", device))
            Bvt[l, b].copy_(_t_recon_t(w, seed, b, l, "v", device))
    return dict(Ak=Ak, Av=Av, Bkt=Bkt, Bvt=Bvt)


def torch_xkv_layer(w: Workload, seed: int, layer: int, device="cuda") -> dict:
    """One layer's slice of torch_xkv_cache (same values): Ak, Av [B][L][r], Bkt, Bvt
    [B][d_kv][r]."""
    import torch
    win = layer // w.window
    return dict(
        Ak=torch.stack([_t_basis(w, seed, b, win, "k", device) for b in range(w.batch)]),
        Av=torch.stack([_t_basis(w, seed, b, win, "v", device) for b in range(w.batch)]),
        Bkt=torch.stack([_t_recon_t(w, seed, b, layer, "k", device) for b in range(w.batch)]),
        Bvt=torch.stack([_t_recon_t(w, seed, b, layer, "v", device) for b in range(w.batch)]))


def torch_needle_chunks(w: Workload, seed: int) -> list:
    return [np_needle_chunks(w, seed, b) for b in range(w.batch)] if w.n_needles else []


def torch_queries(w: Workload, seed: int, cache: dict | None = None, device="cuda"):
    """Query pool q [n_q][N][B][Hq][hd] on a device, with needles planted if the
    workload has them (needle directions from the cache's factors)."""
    import torch
    dt = _tdtype(w.dtype)
    nq = w.q_pool()
    q = torch.empty((nq, w.n_layers, w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32,
                    device=device)
    for s in range(nq):
        for l in range(w.n_layers):
            g = _tgen(seed, "q", s, l, device=device)
            q[s, l] = torch.randn((w.batch, w.n_q_heads, w.head_dim), generator=g,
                                  device=device) * w.head_dim ** -0.25
    if w.n_needles and cache is not None:
        lam = 4.0 * w.head_dim ** 0.25
        C, hd, G = w.chunk, w.head_dim, w.group
        for b, nd in enumerate(torch_needle_chunks(w, seed)):
            for l in range(w.n_layers):
                A = cache["Ak"][l // w.window, b].float()
                abar = torch.stack([A[n * C:(n + 1) * C].mean(0) for n in nd])   # n x r
                Bt = cache["Bkt"][l, b].float()                                   # d_kv x r
                d = (abar @ Bt.T).view(len(nd), w.n_kv_heads, hd)                 # n x H x hd
                u = d / d.norm(dim=-1, keepdim=True)                              # n x H x hd
                pick = torch.tensor([j % len(nd) for j in range(G)], device=device)
                q[:, l, b] += lam * u[pick].permute(1, 0, 2).reshape(-1, hd)[None]
    return q.to(dt)


def torch_layer_queries(w: Workload, seed: int, layer: int, layer_cache: dict, slot: int = 0,
                        device="cuda"):
    """Query slot `slot` of one layer, [B][Hq][hd], as torch_queries builds it (needles
    from the layer's factors)."""
    import torch
    g = _tgen(seed, "q", slot, layer, device=device)
    q = torch.randn((w.batch, w.n_q_heads, w.head_dim), generator=g, device=device) \
        * w.head_dim ** -0.25
    if w.n_needles:
        lam = 4.0 * w.head_dim ** 0.25
        C, hd, G = w.chunk, w.head_dim, w.group
        for b, nd in enumerate(torch_needle_chunks(w, seed)):
            A = layer_cache["Ak"][b].float()
            abar = torch.stack([A[n * C:(n + 1) * C].mean(0) for n in nd])
            d = (abar @ layer_cache["Bkt"][b].float().T).view(len(nd), w.n_kv_heads, hd)
            u = d / d.norm(dim=-1, keepdim=True)                                  # n x H x hd
            pick = torch.tensor([j % len(nd) for j in range(G)], device=device)
            q[b] += lam * u[pick].permute(1, 0, 2).reshape(-1, hd)
    return q.to(_tdtype(w.dtype))


def torch_rcla_cache(w: Workload, seed: int, device="cuda") -> dict:
    """Leader caches with ctx_len valid rows, plus the new-row pool, on a device."""
    import torch
    dt = _tdtype(w.dtype)
    S = leader_set(w)
    nl, B, H, Lm, hd, L = len(S), w.batch, w.n_kv_heads, w.L_max, w.head_dim, w.ctx_len
    K = torch.zeros((nl, B, H, Lm, hd), dtype=dt, device=device)
    V = torch.zeros((nl, B, H, Lm, hd), dtype=dt, device=device)
    for s in range(nl):
        for b in range(B):
            K[s, b, :, :L] = torch.randn((H, L, hd), generator=_tgen(seed, "K", s, b, device=device),
                                         device=device).to(dt)
            V[s, b, :, :L] = torch.randn((H, L, hd), generator=_tgen(seed, "V", s, b, device=device),
                                         device=device).to(dt)
    n_out = int(round(w.outlier_frac * L))
    for b in range(B):
        if n_out:
            g = _tgen(seed, "outlier", b, device=device)
            pos = torch.randperm(L, generator=g, device=device)[:n_out]
            V[:, b, :, pos, :] = (V[:, b, :, pos, :].float() * w.outlier_scale).to(dt)
    nq = w.q_pool()
    kn = torch.randn((nq, nl, B, H, hd), generator=_tgen(seed, "knew", 0, device=device),
                     device=device).to(dt)
    vn = torch.randn((nq, nl, B, H, hd), generator=_tgen(seed, "vnew", 0, device=device),
                     device=device).to(dt)
    return dict(K_lead=K, V_lead=V, k_new=kn, v_new=vn)


def torch_window_caches(W: int, B: int, L: int, d_kv: int, n_modes: int, rank: int,
                        tau: float, gap: float, dtype: str, seed: int, device="cuda"):
    """np_window_caches at full size, built on the device (fp32 QR and products, then
    the storage dtype).  Returns (X [W][B][L][d_kv], s [m] as fp64 numpy)."""
    import torch
    n = W * d_kv
    m = min(n_modes, L, n)
    s = window_spectrum(m, rank, tau, gap)
    st = torch.tensor(s, dtype=torch.float32, device=device)
    X = torch.empty((W, B, L, d_kv), dtype=_tdtype(dtype), device=device)
    for b in range(B):
        gu = _tgen(seed, "clfU", b, device=device)
        gv = _tgen(seed, "clfV", b, device=device)
        U, _ = torch.linalg.qr(torch.randn((L, m), generator=gu, device=device))
        V, _ = torch.linalg.qr(torch.randn((n, m), generator=gv, device=device))
        US = U * st[None, :]
        for l in range(W):
            X[l, b] = (US @ V[l * d_kv:(l + 1) * d_kv].T).to(X.dtype)
    return X, s
