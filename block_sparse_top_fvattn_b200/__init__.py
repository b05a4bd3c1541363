"""Top-p block routing and block-sparse attention for video-DiT layers on B200 (sm_100a).

Thin Python binding of libfvattn.so (include/fvattn.h). PyTorch supplies device memory and
the current stream; every step of the computation runs in the library's CUDA kernels.
There is no CPU or library fallback: if the library is missing, the first call raises.

    csr = route(q, k, p=0.9)                 # q, k: [B, H, S, d] CUDA tensors
    o = sparse_attn(q, k, v, csr)

Method (FVAttn blog summary, section "AI视频生成的阿喀琉斯之踵"): per 64-token query block,
keep the smallest descending-importance set of key blocks whose cumulative softmax mass of
mean-pooled block scores reaches p, then attend exactly over the kept blocks only.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import List, Optional, Tuple

import torch

from . import _lib
from ._lib import (FVATTN_BF16, FVATTN_F32, FVATTN_MODE_FRAME_TOPK, FVATTN_MODE_TOPP, FvattnError, check,
                   load, status_string)

__all__ = ["RouteConfig", "CsrBuffers", "alloc_csr", "route", "route_pool", "route_finish", "sparse_attn",
           "sparse_attn_stamped",
           "sm_busy_imbalance", "block_means", "block_scores", "sparse_attn_timeout_check",
           "block_scores_timeout_check",
           "read_status",
           "workspace_bytes", "shape_of", "load", "FvattnError", "status_string", "rlb_plan", "select_heads",
           "LazyRouter"]

BLOCK = 64


@dataclasses.dataclass
class RouteConfig:
    """Mirror of fvattn_route_cfg (see include/fvattn.h for the meaning of each field)."""
    mode: str = "topp"            # "topp" | "frame_topk" | "topk"
    p: float = 0.9
    force_diag: bool = True
    local_window: int = 0
    frame_len: int = 0
    topk_frames: int = 0
    frame_window: int = -1
    force_first_frame: bool = False
    topk_blocks: int = 0
    sasa_coef: float = 0.0
    sasa_trigger: int = 1
    frame_exact: bool = False

    def to_c(self) -> _lib.RouteCfg:
        mode = {"topp": FVATTN_MODE_TOPP, "frame_topk": FVATTN_MODE_FRAME_TOPK,
                "topk": _lib.FVATTN_MODE_TOPK_BLOCKS}[self.mode]
        return _lib.RouteCfg(mode, float(self.p), int(self.force_diag), int(self.local_window), int(self.frame_len),
                             int(self.topk_frames), int(self.frame_window), int(self.force_first_frame),
                             int(self.topk_blocks), float(self.sasa_coef), int(self.sasa_trigger),
                             int(self.frame_exact))


@dataclasses.dataclass
class CsrBuffers:
    """Router outputs (device tensors) in the layout of fvattn_csr."""
    row_ptr: torch.Tensor      # int32 [BH*nb + 1]
    col_idx: torch.Tensor      # int32 [BH*nb*nb]
    head_load: torch.Tensor    # int64 [BH]
    tile_cost: torch.Tensor    # int32 [BH*ceil(nb/2)]
    tile_order: torch.Tensor   # int32 [BH*ceil(nb/2)]
    nnz: torch.Tensor          # int64 [1]
    status: torch.Tensor       # int32 [4]
    B: int
    H: int
    S: int
    col_code: Optional[torch.Tensor] = None   # int32 [BH*nb*nb]: per-entry token masks (frame_exact)

    @property
    def nb(self) -> int:
        return -(-self.S // BLOCK)

    def to_c(self) -> _lib.Csr:
        return _lib.Csr(self.row_ptr.data_ptr(), self.col_idx.data_ptr(), self.col_idx.numel(),
                        self.head_load.data_ptr(), self.tile_cost.data_ptr(), self.tile_order.data_ptr(),
                        self.nnz.data_ptr(), self.status.data_ptr(),
                        self.col_code.data_ptr() if self.col_code is not None else None)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FVATTN_BF16
    if t.dtype == torch.float32:
        return FVATTN_F32
    raise TypeError(f"unsupported dtype {t.dtype}; bf16 or fp32")


def shape_of(q: torch.Tensor, scale: float = 0.0) -> _lib.Shape:
    if q.dim() != 4:
        raise ValueError("expected [B, H, S, d]")
    B, H, S, d = q.shape
    return _lib.Shape(B, H, S, d, BLOCK, _dtype_code(q), float(scale))


def _stream(stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check_tensor(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous [B, H, S, d]")


def alloc_csr(B: int, H: int, S: int, device="cuda", codes: bool = False) -> CsrBuffers:
    """Router output buffers; `codes` adds the per-entry token masks that token-exact frame
    mode (RouteConfig.frame_exact) writes and the attention applies."""
    nb = -(-S // BLOCK)
    nt = B * H * (-(-nb // 2))
    i32, i64 = torch.int32, torch.int64
    return CsrBuffers(
        col_code=torch.empty(B * H * nb * nb, dtype=i32, device=device) if codes else None,
        row_ptr=torch.empty(B * H * nb + 1, dtype=i32, device=device),
        col_idx=torch.empty(B * H * nb * nb, dtype=i32, device=device),
        head_load=torch.empty(B * H, dtype=i64, device=device),
        tile_cost=torch.empty(nt, dtype=i32, device=device),
        tile_order=torch.empty(nt, dtype=i32, device=device),
        nnz=torch.empty(1, dtype=i64, device=device),
        status=torch.zeros(4, dtype=i32, device=device),
        B=B, H=H, S=S)


def workspace_bytes(q: torch.Tensor, cfg: RouteConfig) -> int:
    n = load().fvattn_route_workspace_bytes(ctypes.byref(shape_of(q)), ctypes.byref(cfg.to_c()))
    if n == 0:
        raise FvattnError(_lib.FVATTN_ERR_INVALID, "fvattn_route_workspace_bytes")
    return int(n)


def route(q: torch.Tensor, k: torch.Tensor, cfg: Optional[RouteConfig] = None, *, p: Optional[float] = None,
          csr: Optional[CsrBuffers] = None, workspace: Optional[torch.Tensor] = None,
          stream: Optional[torch.cuda.Stream] = None, scale: float = 0.0) -> CsrBuffers:
    """Run fvattn_route on the current (or given) stream. Returns the CSR buffers."""
    cfg = cfg or RouteConfig()
    if p is not None:
        cfg = dataclasses.replace(cfg, p=p)
    _check_tensor(q, "q")
    _check_tensor(k, "k")
    if k.shape != q.shape or k.dtype != q.dtype:
        raise ValueError("q and k must have the same shape and dtype")
    B, H, S, _ = q.shape
    if csr is None:
        csr = alloc_csr(B, H, S, q.device, codes=cfg.frame_exact)
    elif cfg.frame_exact and csr.col_code is None:
        raise ValueError("token-exact frame mode needs CSR buffers with col_code (alloc_csr(..., codes=True))")
    shp = shape_of(q, scale)
    c_cfg = cfg.to_c()
    nws = workspace_bytes(q, cfg)
    if workspace is None or workspace.numel() < nws:
        workspace = torch.empty(nws, dtype=torch.uint8, device=q.device)
    c_csr = csr.to_c()
    check(load().fvattn_route(q.data_ptr(), k.data_ptr(), ctypes.byref(shp), ctypes.byref(c_cfg),
                              ctypes.byref(c_csr), workspace.data_ptr(), nws, _stream(stream)), "fvattn_route")
    csr._workspace = workspace      # keep the scratch alive until the kernels have run
    return csr


def route_pool(q: torch.Tensor, k: torch.Tensor, cfg: RouteConfig, block_begin: int, block_end: int,
               workspace: torch.Tensor, *, stream: Optional[torch.cuda.Stream] = None, scale: float = 0.0) -> None:
    """fvattn_route_pool: step 1 of the router for the 64-token blocks [block_begin, block_end)
    of every head of q, k ([B, H, S, d]; only those blocks' tokens are read) into `workspace`
    (uint8, at least workspace_bytes(q, cfg))."""
    _check_tensor(q, "q")
    _check_tensor(k, "k")
    if k.shape != q.shape or k.dtype != q.dtype:
        raise ValueError("q and k must have the same shape and dtype")
    nws = workspace_bytes(q, cfg)
    if workspace.numel() < nws or not workspace.is_cuda:
        raise ValueError(f"workspace needs {nws} bytes on the device")
    check(load().fvattn_route_pool(q.data_ptr(), k.data_ptr(), ctypes.byref(shape_of(q, scale)),
                                   ctypes.byref(cfg.to_c()), int(block_begin), int(block_end), workspace.data_ptr(),
                                   nws, _stream(stream)), "fvattn_route_pool")


def route_finish(q: torch.Tensor, cfg: RouteConfig, workspace: torch.Tensor, *, csr: Optional[CsrBuffers] = None,
                 stream: Optional[torch.cuda.Stream] = None, scale: float = 0.0) -> CsrBuffers:
    """fvattn_route_finish: steps 2 and 3 of the router from a workspace in which route_pool has
    pooled every block of every head (q gives the shape only). Returns the CSR buffers."""
    _check_tensor(q, "q")
    B, H, S, _ = q.shape
    if csr is None:
        csr = alloc_csr(B, H, S, q.device, codes=cfg.frame_exact)
    nws = workspace_bytes(q, cfg)
    if workspace.numel() < nws or not workspace.is_cuda:
        raise ValueError(f"workspace needs {nws} bytes on the device")
    check(load().fvattn_route_finish(ctypes.byref(shape_of(q, scale)), ctypes.byref(cfg.to_c()),
                                     ctypes.byref(csr.to_c()), workspace.data_ptr(), nws, _stream(stream)),
          "fvattn_route_finish")
    csr._workspace = workspace
    return csr


def sparse_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, csr: CsrBuffers, *,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None, scale: float = 0.0) -> torch.Tensor:
    """Run fvattn_sparse_attn: exact attention over the routed key blocks. Returns O."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_tensor(t, n)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v must have the same shape and dtype")
    if out is None:
        out = torch.empty_like(q)
    shp = shape_of(q, scale)
    c_csr = csr.to_c()
    check(load().fvattn_sparse_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(shp), ctypes.byref(c_csr),
                                    out.data_ptr(), lse.data_ptr() if lse is not None else None, _stream(stream)),
          "fvattn_sparse_attn")
    return out


def sparse_attn_stamped(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, csr: CsrBuffers, *,
                        out: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                        scale: float = 0.0):
    """fvattn_sparse_attn_stamped (bf16): the attention plus, per CTA of its persistent grid, the
    SM id and the busy interval in ns. Returns (O, stamps [n_cta, 3] int64 on the device)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_tensor(t, n)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v must have the same shape and dtype")
    if out is None:
        out = torch.empty_like(q)
    shp = shape_of(q, scale)
    lib = load()
    words = lib.fvattn_attn_stamp_words(ctypes.byref(shp))
    if words <= 0:
        raise FvattnError(_lib.FVATTN_ERR_UNSUPPORTED, "fvattn_attn_stamp_words")
    stamps = torch.zeros(words, dtype=torch.int64, device=q.device)
    check(lib.fvattn_sparse_attn_stamped(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(shp),
                                         ctypes.byref(csr.to_c()), out.data_ptr(), None, stamps.data_ptr(), words,
                                         _stream(stream)), "fvattn_sparse_attn_stamped")
    return out, stamps.view(-1, 3)


def sm_busy_imbalance(stamps: torch.Tensor) -> dict:
    """From the [n_cta, 3] stamps of sparse_attn_stamped: each SM's busy time (last end minus
    first start over its CTAs), and max / mean of those over the SMs."""
    st = stamps.cpu().numpy().astype("int64")
    busy = {}
    for sm, t0, t1 in st:
        lo, hi = busy.get(int(sm), (t0, t1))
        busy[int(sm)] = (min(lo, t0), max(hi, t1))
    times = [hi - lo for lo, hi in busy.values()]
    mean = sum(times) / len(times)
    return {"sms": len(times), "max_ns": int(max(times)), "mean_ns": float(mean),
            "imbalance": float(max(times) / mean) if mean > 0 else 1.0}


def block_means(x: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """fp64 means of every 64-token block of x ([B, H, S, d]) over its valid tokens."""
    _check_tensor(x, "x")
    B, H, S, d = x.shape
    out = torch.empty((B, H, -(-S // BLOCK), d), dtype=torch.float64, device=x.device)
    check(load().fvattn_block_means(x.data_ptr(), ctypes.byref(shape_of(x)), out.data_ptr(), _stream(stream)),
          "fvattn_block_means")
    return out


def block_scores(q: torch.Tensor, k: torch.Tensor, scale: float = 0.0,
                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """fvattn_block_scores: the router's fp64 block scores <Qbar_i, Kbar_j> * scale of every head,
    as a [B, H, nb, nb] view of the library's [B*H*nb, ld] output (scale 0: 1/sqrt(d)). Raises
    FvattnError if a kernel reported an error."""
    _check_tensor(q, "q")
    _check_tensor(k, "k")
    if k.shape != q.shape or k.dtype != q.dtype or k.device != q.device:
        raise ValueError("q and k must have the same shape, dtype and device")
    B, H, S, d = q.shape
    shp = shape_of(q, scale)
    lib = load()
    nws = lib.fvattn_block_scores_workspace_bytes(ctypes.byref(shp))
    ld = lib.fvattn_block_scores_ld(ctypes.byref(shp))
    if nws == 0 or ld == 0:
        raise FvattnError(_lib.FVATTN_ERR_INVALID, "fvattn_block_scores_workspace_bytes")
    nb = -(-S // BLOCK)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device)
    out = torch.empty((B * H * nb, ld), dtype=torch.float64, device=q.device)
    status = torch.zeros(4, dtype=torch.int32, device=q.device)
    check(lib.fvattn_block_scores(q.data_ptr(), k.data_ptr(), ctypes.byref(shp), out.data_ptr(), ws.data_ptr(), nws,
                                  status.data_ptr(), _stream(stream)), "fvattn_block_scores")
    (stream if stream is not None else torch.cuda.current_stream(q.device)).synchronize()
    code = int(status[0].item())
    if code != 0:
        raise FvattnError(code, "fvattn_block_scores (device status)")
    return out.view(B, H, nb, ld)[..., :nb]


def sparse_attn_timeout_check(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, csr: CsrBuffers, out: torch.Tensor,
                              polls: int = 64, stream: Optional[torch.cuda.Stream] = None) -> int:
    """fvattn_sparse_attn_timeout_check: the attention kernel with a first bounded wait on a
    barrier that nothing completes, so that it times out before any copy or MMA. Returns the
    device status word afterwards (FVATTN_ERR_TIMEOUT expected); `out` is left unwritten."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check_tensor(t, n)
    lib = load()
    check(lib.fvattn_sparse_attn_timeout_check(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(shape_of(q)),
                                               ctypes.byref(csr.to_c()), out.data_ptr(), int(polls), _stream(stream)),
          "fvattn_sparse_attn_timeout_check")
    return read_status(csr, stream)


def block_scores_timeout_check(q: torch.Tensor, k: torch.Tensor, polls: int = 64,
                               stream: Optional[torch.cuda.Stream] = None) -> Tuple[int, torch.Tensor]:
    """fvattn_block_scores_timeout_check: the block-score kernel with a first bounded wait on a
    barrier that nothing completes. Returns (device status word, the score buffer, filled with NaN
    before the call and left unwritten by the kernel)."""
    _check_tensor(q, "q")
    _check_tensor(k, "k")
    B, H, S, d = q.shape
    shp = shape_of(q)
    lib = load()
    nws = lib.fvattn_block_scores_workspace_bytes(ctypes.byref(shp))
    ld = lib.fvattn_block_scores_ld(ctypes.byref(shp))
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device)
    out = torch.full((B * H * -(-S // BLOCK), ld), float("nan"), dtype=torch.float64, device=q.device)
    status = torch.zeros(4, dtype=torch.int32, device=q.device)
    check(lib.fvattn_block_scores_timeout_check(q.data_ptr(), k.data_ptr(), ctypes.byref(shp), out.data_ptr(),
                                                ws.data_ptr(), nws, status.data_ptr(), int(polls), _stream(stream)),
          "fvattn_block_scores_timeout_check")
    (stream if stream is not None else torch.cuda.current_stream(q.device)).synchronize()
    return int(status[0].item()), out


def read_status(csr: CsrBuffers, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise the stream and return the device status word (0 = ok)."""
    return int(load().fvattn_read_status(ctypes.byref(csr.to_c()), _stream(stream)))


def select_heads(csr: CsrBuffers, active: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """fvattn_select_heads: restrict the next sparse_attn on `csr` to the heads bh with
    active[bh] != 0 (active: CUDA uint8/bool tensor [B*H]). The next route on `csr` undoes it."""
    if not active.is_cuda or active.numel() != csr.B * csr.H:
        raise ValueError("active must be a CUDA tensor of B*H flags")
    act = active.to(torch.uint8).contiguous()
    shp = _lib.Shape(csr.B, csr.H, csr.S, 64, BLOCK, FVATTN_BF16, 0.0)    # only B, H, S are read
    check(load().fvattn_select_heads(ctypes.byref(shp), ctypes.byref(csr.to_c()), act.data_ptr(), _stream(stream)),
          "fvattn_select_heads")
    csr._active = act                 # keep the flags alive until the kernel has run


def rlb_plan(loads, target: float = 1.05, max_moves_per_rank: int = 1) -> Tuple[List[Tuple[int, int, int]], List[int]]:
    """fvattn_rlb_plan on a [ranks, heads_per_rank] array of per-head loads (host). Returns the
    moves (sender rank, sender's local head, receiver rank) in plan order and the rank loads
    after them."""
    import numpy as np
    L = np.ascontiguousarray(np.asarray(loads, dtype=np.int64))
    if L.ndim != 2:
        raise ValueError("loads must be [ranks, heads_per_rank]")
    R, Hl = L.shape
    cap = max(1, R * min(max_moves_per_rank, Hl))
    moves = np.zeros(3 * cap, dtype=np.int32)
    rl = np.zeros(R, dtype=np.int64)
    n = ctypes.c_int32(0)
    check(load().fvattn_rlb_plan(L.ctypes.data, R, Hl, float(target), int(max_moves_per_rank), moves.ctypes.data, cap,
                                 ctypes.byref(n), rl.ctypes.data), "fvattn_rlb_plan")
    mv = moves[: 3 * n.value].reshape(-1, 3)
    return [(int(a), int(b), int(c)) for a, b, c in mv], [int(x) for x in rl]


class LazyRouter:
    """Routing reuse across diffusion steps for one attention layer: the block selection (and
    its tile schedule) is recomputed only every `refresh_every` steps and reused in between
    (the video-generation acceleration notes' "lazy" mask update, e.g. every 4 diffusion
    steps, to save the cost of generating the mask). Holds the layer's CSR and workspace.

        layer = LazyRouter(RouteConfig(p=0.9), refresh_every=4)
        for step in range(n_steps):
            o = layer(q, k, v, step)
    """

    def __init__(self, cfg: Optional[RouteConfig] = None, refresh_every: int = 4):
        if refresh_every < 1:
            raise ValueError("refresh_every must be >= 1")
        self.cfg = cfg or RouteConfig()
        self.refresh_every = int(refresh_every)
        self.csr: Optional[CsrBuffers] = None
        self.workspace: Optional[torch.Tensor] = None
        self.last_refresh: Optional[int] = None
        self.routed = 0

    def should_refresh(self, step: int, shape) -> bool:
        if self.csr is None or self.last_refresh is None:
            return True
        if (self.csr.B, self.csr.H, self.csr.S) != tuple(shape[:3]):
            return True
        return step < self.last_refresh or step - self.last_refresh >= self.refresh_every

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, step: int, *,
                 out: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        if self.should_refresh(step, q.shape):
            B, H, S, _ = q.shape
            if self.csr is None or (self.csr.B, self.csr.H, self.csr.S) != (B, H, S):
                self.csr = alloc_csr(B, H, S, q.device, codes=self.cfg.frame_exact)
                self.workspace = None
            route(q, k, self.cfg, csr=self.csr, workspace=self.workspace, stream=stream)
            self.workspace = self.csr._workspace
            self.last_refresh = step
            self.routed += 1
        return sparse_attn(q, k, v, self.csr, out=out, stream=stream)
