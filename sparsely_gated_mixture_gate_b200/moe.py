"""Thin Python binding of the C ABI: argument marshalling over torch device
memory and the current CUDA stream.  Every step of the layer runs in the CUDA
library; this module only allocates outputs / workspace with torch and passes
pointers.  There is no CPU path: calls fail loudly when the library or a CUDA
device is missing.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import math
from typing import Optional

import torch

from . import _lib
from ._lib import moe_config, moe_expert_params, moe_gate_params


class MoEError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != _lib.MOE_OK:
        msg = _lib.load().moe_strerror(rc).decode()
        raise MoEError(f"{what}: {msg} ({rc})")


@dataclasses.dataclass
class Config:
    """Mirror of ``moe_config`` (include/moe.h)."""
    T: int
    d: int
    n: int
    k: int
    f: int
    hier_a: int = 0
    hier_b: int = 0
    hier_k1: int = 0
    hier_k2: int = 0
    router: int = 0
    noise: int = 1
    expert_bf16: int = 1
    seed: int = 0
    capacity_factor: float = 0.0
    passthrough: int = 0
    w_importance: float = 0.1
    w_load: float = 0.1
    alpha: float = 0.01
    gate_precision: int = 0   # 0: fp32 multiply-adds, 1: tensor cores, 3-pass TF32 split
    shared_expert: int = 0    # 1: one always-active expert (W1s, b1s, W2s, b2s) in forward
    router_stats: int = 0     # 1: forward reports the router z-loss and entropy (losses[8:10])
    backward: int = 0         # 1: the layer also runs the backward pass (workspace, saved state)
    w_z: float = 0.0          # backward: weight of the router z-loss (losses[8])
    w_entropy: float = 0.0    # backward: weight rewarding the gate entropy (-losses[9])
    token_base: int = 0       # first token's index in the noise counter (a shard of a batch)

    @classmethod
    def from_workload(cls, w, T: Optional[int] = None) -> "Config":
        kw = {f.name: getattr(w, f.name) for f in dataclasses.fields(cls) if hasattr(w, f.name)}
        if T is not None:
            kw["T"] = T
        return cls(**kw)

    def c(self) -> moe_config:
        return moe_config(T=self.T, d=self.d, n=self.n, k=self.k, f=self.f, hier_a=self.hier_a,
                          hier_b=self.hier_b, hier_k1=self.hier_k1, hier_k2=self.hier_k2,
                          router=self.router, noise=self.noise,
                          expert_dtype=_lib.BF16 if self.expert_bf16 else _lib.F32,
                          seed=self.seed, capacity_factor=float(self.capacity_factor),
                          overflow_passthrough=self.passthrough, w_importance=self.w_importance,
                          w_load=self.w_load, alpha_aux=self.alpha,
                          gate_precision=self.gate_precision, shared_expert=self.shared_expert,
                          router_stats=self.router_stats, backward=self.backward,
                          w_z=self.w_z, w_entropy=self.w_entropy, token_base=self.token_base)

    @property
    def expert_dtype(self):
        return torch.bfloat16 if self.expert_bf16 else torch.float32


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(device) -> torch.device:
    d = torch.device(device)
    if d.type == "cuda" and d.index is None:
        d = torch.device("cuda", torch.cuda.current_device())
    return d


def _need(t: Optional[torch.Tensor], name: str, dtype, shape=None, device=None, optional=False):
    if t is None:
        if optional:
            return
        raise MoEError(f"{name} is required")
    if not t.is_cuda:
        raise MoEError(f"{name} must be a CUDA tensor (the layer has no CPU path)")
    if t.dtype != dtype:
        raise MoEError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise MoEError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise MoEError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != _dev(device):
        raise MoEError(f"{name} is on {t.device}, expected {device}")


def validate(cfg: Config) -> bool:
    c = cfg.c()
    return _lib.load().moe_validate(C.byref(c)) == _lib.MOE_OK


def workspace_size(cfg: Config) -> int:
    c = cfg.c()
    out = C.c_size_t(0)
    _check(_lib.load().moe_workspace_size(C.byref(c), C.byref(out)), "moe_workspace_size")
    return int(out.value)


def capacity(cfg: Config) -> int:
    c = cfg.c()
    out = C.c_int64(0)
    _check(_lib.load().moe_capacity(C.byref(c), C.byref(out)), "moe_capacity")
    return int(out.value)


def workspace(cfg: Config, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(workspace_size(cfg), 256), dtype=torch.uint8, device=device)


def gate_params(params: dict, seed_dev: Optional[torch.Tensor] = None) -> moe_gate_params:
    return moe_gate_params(W_g=_ptr(params.get("Wg")), b_g=_ptr(params.get("bg")),
                           W_noise=_ptr(params.get("Wn")), W_g2=_ptr(params.get("Wg2")),
                           b_g2=_ptr(params.get("bg2")), W_noise2=_ptr(params.get("Wn2")),
                           sel_bias=_ptr(params.get("sel_bias")), seed_dev=_ptr(seed_dev))


def noise_step(seed_dev: torch.Tensor):
    """Advance the device noise key by one on the current stream."""
    _need(seed_dev, "seed_dev", torch.int64, (1,))
    _check(_lib.load().moe_noise_step(_ptr(seed_dev), _stream()), "moe_noise_step")


def expert_params(params: dict) -> moe_expert_params:
    return moe_expert_params(W1=_ptr(params.get("W1")), b1=_ptr(params.get("b1")),
                             W2=_ptr(params.get("W2")), b2=_ptr(params.get("b2")),
                             W1s=_ptr(params.get("W1s")), b1s=_ptr(params.get("b1s")),
                             W2s=_ptr(params.get("W2s")), b2s=_ptr(params.get("b2s")))


def _check_params(cfg: Config, p: dict, dev, gate=True, experts=True):
    gn = cfg.hier_a if cfg.hier_a else cfg.n
    if gate:
        _need(p.get("Wg"), "Wg", torch.float32, (cfg.d, gn), dev)
        _need(p.get("Wn"), "Wn", torch.float32, (cfg.d, gn), dev, optional=not cfg.noise)
        _need(p.get("bg"), "bg", torch.float32, (gn,), dev, optional=True)
        if cfg.router == 2:
            _need(p.get("sel_bias"), "sel_bias", torch.float32, (cfg.n,), dev, optional=True)
        if cfg.hier_a:
            sh = (cfg.hier_a, cfg.d, cfg.hier_b)
            _need(p.get("Wg2"), "Wg2", torch.float32, sh, dev)
            _need(p.get("Wn2"), "Wn2", torch.float32, sh, dev, optional=not cfg.noise)
            _need(p.get("bg2"), "bg2", torch.float32, (cfg.hier_a, cfg.hier_b), dev, optional=True)
    if experts:
        _need(p.get("W1"), "W1", cfg.expert_dtype, (cfg.n, cfg.f, cfg.d), dev)
        _need(p.get("W2"), "W2", cfg.expert_dtype, (cfg.n, cfg.d, cfg.f), dev)
        _need(p.get("b1"), "b1", torch.float32, (cfg.n, cfg.f), dev, optional=True)
        _need(p.get("b2"), "b2", torch.float32, (cfg.n, cfg.d), dev, optional=True)
        if cfg.shared_expert:
            _need(p.get("W1s"), "W1s", cfg.expert_dtype, (cfg.f, cfg.d), dev)
            _need(p.get("W2s"), "W2s", cfg.expert_dtype, (cfg.d, cfg.f), dev)
            _need(p.get("b1s"), "b1s", torch.float32, (cfg.f,), dev, optional=True)
            _need(p.get("b2s"), "b2s", torch.float32, (cfg.d,), dev, optional=True)


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def status_bits(status: torch.Tensor) -> int:
    return int(status.item())


# ---------------------------------------------------------------- step calls
def gate(cfg: Config, x: torch.Tensor, params: dict, ws=None, status=None):
    dev = x.device
    _need(x, "x", torch.float32, (cfg.T, cfg.d))
    _check_params(cfg, params, dev, experts=False)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    g = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    load = torch.empty(cfg.n, dtype=torch.float32, device=dev)
    psum = torch.empty(cfg.n, dtype=torch.float32, device=dev)
    ws = workspace(cfg, dev) if ws is None else ws
    status = new_status(dev) if status is None else status
    c = cfg.c()
    gp = gate_params(params)
    _check(_lib.load().moe_gate(C.byref(c), _ptr(x), C.byref(gp), _ptr(idx), _ptr(g), _ptr(load),
                                _ptr(psum), _ptr(ws), ws.numel(), _ptr(status), _stream()), "moe_gate")
    return dict(topk_idx=idx, topk_gate=g, load=load, prob_sum=psum, status=status)


def dispatch(cfg: Config, x: Optional[torch.Tensor], topk_idx: torch.Tensor, ws=None, status=None):
    dev = topk_idx.device
    _need(topk_idx, "topk_idx", torch.int32, (cfg.T, cfg.k))
    if x is not None:
        _need(x, "x", torch.float32, (cfg.T, cfg.d), dev)
    S = cfg.T * cfg.k
    counts = torch.empty(cfg.n, dtype=torch.int32, device=dev)
    offsets = torch.empty(cfg.n + 1, dtype=torch.int32, device=dev)
    perm_token = torch.full((max(S, 1),), -1, dtype=torch.int32, device=dev)
    row_of = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(max(S, 1), cfg.d, dtype=cfg.expert_dtype, device=dev) if x is not None else None
    ws = workspace(cfg, dev) if ws is None else ws
    status = new_status(dev) if status is None else status
    c = cfg.c()
    _check(_lib.load().moe_dispatch(C.byref(c), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                    _ptr(perm_token), _ptr(row_of), _ptr(x_perm), _ptr(ws), ws.numel(),
                                    _ptr(status), _stream()), "moe_dispatch")
    return dict(counts=counts, offsets=offsets, perm_token=perm_token, row_of=row_of, x_perm=x_perm,
                status=status)


def expert_ffn(cfg: Config, x_perm: torch.Tensor, offsets: torch.Tensor, params: dict, ws=None,
               status=None):
    dev = x_perm.device
    S = cfg.T * cfg.k
    _need(x_perm, "x_perm", cfg.expert_dtype, (max(S, 1), cfg.d))
    _need(offsets, "offsets", torch.int32, (cfg.n + 1,), dev)
    _check_params(cfg, params, dev, gate=False)
    y_perm = torch.empty(max(S, 1), cfg.d, dtype=cfg.expert_dtype, device=dev)
    ws = workspace(cfg, dev) if ws is None else ws
    status = new_status(dev) if status is None else status
    c = cfg.c()
    ep = expert_params(params)
    _check(_lib.load().moe_expert_ffn(C.byref(c), _ptr(x_perm), _ptr(offsets), C.byref(ep), _ptr(y_perm),
                                      _ptr(ws), ws.numel(), _ptr(status), _stream()), "moe_expert_ffn")
    return dict(y_perm=y_perm, status=status)


def combine(cfg: Config, y_perm: torch.Tensor, topk_gate: torch.Tensor, row_of: torch.Tensor,
            x: Optional[torch.Tensor] = None, status=None):
    dev = y_perm.device
    _need(y_perm, "y_perm", cfg.expert_dtype, None)
    _need(topk_gate, "topk_gate", torch.float32, (cfg.T, cfg.k), dev)
    _need(row_of, "row_of", torch.int32, (cfg.T, cfg.k), dev)
    if x is not None:
        _need(x, "x", torch.float32, (cfg.T, cfg.d), dev)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    status = new_status(dev) if status is None else status
    c = cfg.c()
    _check(_lib.load().moe_combine(C.byref(c), _ptr(y_perm), _ptr(topk_gate), _ptr(row_of), _ptr(x),
                                   _ptr(y), _ptr(status), _stream()), "moe_combine")
    return dict(y=y, status=status)


def balance_losses(cfg: Config, topk_idx, topk_gate, counts, load, prob_sum=None, ws=None, status=None):
    dev = topk_idx.device
    importance = torch.empty(cfg.n, dtype=torch.float32, device=dev)
    losses = torch.empty(10, dtype=torch.float32, device=dev)
    ws = workspace(cfg, dev) if ws is None else ws
    status = new_status(dev) if status is None else status
    c = cfg.c()
    _check(_lib.load().moe_balance_losses(C.byref(c), _ptr(topk_idx), _ptr(topk_gate), _ptr(counts),
                                          _ptr(load), _ptr(prob_sum), _ptr(importance), _ptr(losses),
                                          _ptr(ws), ws.numel(), _ptr(status), _stream()),
           "moe_balance_losses")
    return dict(importance=importance, losses=losses, status=status)


def gather_rows(src: torch.Tensor, index: torch.Tensor, src_rows: Optional[int] = None,
                out: Optional[torch.Tensor] = None, status=None) -> torch.Tensor:
    """out[i] = src[index[i]] (whole rows, through moe_gather_rows); an index
    outside [0, src_rows) gives a zero row and the BAD_INDEX status bit."""
    _need(index, "index", torch.int32, None, src.device)
    rows = index.numel()
    if not src.is_cuda or not src.is_contiguous():
        raise MoEError("src must be a contiguous CUDA tensor")
    row_shape = tuple(src.shape[1:])
    if out is None:
        out = torch.empty((rows,) + row_shape, dtype=src.dtype, device=src.device)
    row_bytes = math.prod(row_shape) * src.element_size()
    status = new_status(src.device) if status is None else status
    _check(_lib.load().moe_gather_rows(_ptr(src), _ptr(index), _ptr(out), rows, row_bytes,
                                       src.shape[0] if src_rows is None else src_rows,
                                       _ptr(status), _stream()), "moe_gather_rows")
    return out


def balance_from_totals(cfg: Config, importance, load, counts, prob_sum, dropped, status=None):
    """The losses [10] of a batch from its totals over data-parallel shards
    (moe_balance_from_totals; cfg.T is the whole batch)."""
    dev = importance.device
    losses = torch.empty(10, dtype=torch.float32, device=dev)
    status = new_status(dev) if status is None else status
    c = cfg.c()
    _check(_lib.load().moe_balance_from_totals(C.byref(c), _ptr(importance), _ptr(load), _ptr(counts),
                                               _ptr(prob_sum), _ptr(dropped), _ptr(losses),
                                               _ptr(status), _stream()), "moe_balance_from_totals")
    return losses


# ---------------------------------------------------------------- fused layer
class MoELayer:
    """Parameters plus pre-allocated workspace and outputs for repeated calls
    of the fused ``moe_forward`` on one device.

    Noise: the noisy gate draws a new StandardNormal() every time it runs.
    The layer keeps its noise key in a device word that every forward step
    (direct or replayed from a CUDA graph) first advances by one, so step s
    of the layer draws with key cfg.seed + s, and a backward step uses the key
    of the forward before it.  noise_seed_(v) makes the next step draw with
    key v.  With resample_noise=False every step draws with cfg.seed."""

    def __init__(self, cfg: Config, params: dict, device=None, resample_noise: bool = True):
        self.cfg = cfg
        self.params = params
        dev = _dev(device) if device is not None else params["Wg"].device
        self.device = dev
        _check_params(cfg, params, dev)
        _lib.load()
        self._c = cfg.c()
        self.resample_noise = bool(resample_noise) and bool(cfg.noise)
        # the key the last step used (the next step adds one first); uint64 bits in an int64
        self.seed_dev = torch.empty(1, dtype=torch.int64, device=dev)
        self.noise_seed_(cfg.seed)
        self._gp = gate_params(params, self.seed_dev)
        self._ep = expert_params(params)
        self.ws = workspace(cfg, dev)
        self.status = new_status(dev)
        T, k, n, d = cfg.T, cfg.k, cfg.n, cfg.d
        self.y = torch.empty(T, d, dtype=torch.float32, device=dev)
        self.topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.topk_gate = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.importance = torch.empty(n, dtype=torch.float32, device=dev)
        self.load = torch.empty(n, dtype=torch.float32, device=dev)
        self.counts = torch.empty(n, dtype=torch.int32, device=dev)
        self.losses = torch.empty(10, dtype=torch.float32, device=dev)

    def noise_seed_(self, seed: int):
        """The next forward step draws its noise with key ``seed`` (stream
        ordered: a device write on the current stream)."""
        first = (seed - 1) if self.resample_noise else seed
        first &= (1 << 64) - 1
        self.seed_dev.fill_(first - (1 << 64) if first >= (1 << 63) else first)

    def forward_(self, x: torch.Tensor, stream=None, y: Optional[torch.Tensor] = None,
                 losses: Optional[torch.Tensor] = None):
        """Run the layer on device-resident x; outputs land in this object's
        buffers, or in y / losses when given (asynchronous on the stream).
        Advances the noise key first (see the class notes)."""
        _need(x, "x", torch.float32, (self.cfg.T, self.cfg.d), self.device)
        y = self.y if y is None else y
        losses = self.losses if losses is None else losses
        st = C.c_void_p(stream.cuda_stream) if stream is not None else _stream()
        if self.resample_noise:
            _check(_lib.load().moe_noise_step(_ptr(self.seed_dev), st), "moe_noise_step")
        _check(_lib.load().moe_forward(C.byref(self._c), _ptr(x), C.byref(self._gp), C.byref(self._ep),
                                       _ptr(y), _ptr(self.topk_idx), _ptr(self.topk_gate),
                                       _ptr(self.importance), _ptr(self.load), _ptr(self.counts),
                                       _ptr(losses), _ptr(self.ws), self.ws.numel(),
                                       _ptr(self.status), st), "moe_forward")
        return y

    def _graph(self, key, record):
        """The CUDA graph captured for these buffers (key), captured on first
        use: record() issues the calls on the given stream, once outside the
        capture (one-time set-up) and once inside it."""
        graphs = self.__dict__.setdefault("_graphs", {})
        g = graphs.get(key)
        if g is None:
            cap = torch.cuda.Stream(device=self.device)
            cap.wait_stream(torch.cuda.current_stream(self.device))
            with torch.cuda.stream(cap):
                seed = self.seed_dev.clone()
                record(cap)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                record(cap)
            with torch.cuda.stream(cap):
                # the set-up call consumed a noise key: put it back, so the
                # replay that follows draws what a direct call would have
                self.seed_dev.copy_(seed)
            torch.cuda.current_stream(self.device).wait_stream(cap)
            graphs[key] = g
        return g

    def forward_graph_(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                       losses: Optional[torch.Tensor] = None) -> torch.Tensor:
        """forward_ replayed from a CUDA graph on the current stream.  A graph
        is captured on the first call for each set of buffers (x, y, losses;
        their addresses are baked in, their contents may change between
        calls); the library's launches, the side stream's fork and join and
        its memsets are all captured, so a replay runs the same kernels on the
        same buffers with one host call."""
        _need(x, "x", torch.float32, (self.cfg.T, self.cfg.d), self.device)
        y = self.y if y is None else y
        losses = self.losses if losses is None else losses
        g = self._graph(("fwd", x.data_ptr(), y.data_ptr(), losses.data_ptr()),
                        lambda st: self.forward_(x, stream=st, y=y, losses=losses))
        g.replay()
        return y

    def train_graph_(self, x: torch.Tensor, dy: torch.Tensor, y: Optional[torch.Tensor] = None,
                     losses: Optional[torch.Tensor] = None,
                     dx: Optional[torch.Tensor] = None) -> dict:
        """forward_ then backward_ replayed from one CUDA graph on the current
        stream, captured on the first call for each set of buffers (x, dy, y,
        losses, dx)."""
        _need(x, "x", torch.float32, (self.cfg.T, self.cfg.d), self.device)
        _need(dy, "dy", torch.float32, (self.cfg.T, self.cfg.d), self.device)
        grads = self.grads()
        y = self.y if y is None else y
        losses = self.losses if losses is None else losses
        dx = grads["dx"] if dx is None else dx

        def record(st):
            self.forward_(x, stream=st, y=y, losses=losses)
            self.backward_(x, dy, stream=st, dx=dx)
        g = self._graph(("train", x.data_ptr(), dy.data_ptr(), y.data_ptr(), losses.data_ptr(),
                         dx.data_ptr()), record)
        g.replay()
        return grads

    def release_graph(self):
        """Drop the captured graphs."""
        self.__dict__["_graphs"] = {}

    def grads(self, intermediates: bool = False) -> dict:
        """Gradient buffers of this layer (allocated on first use), fp32 in
        the parameters' layouts; with intermediates also dgate [T][k] and,
        for a flat layer, dlogits [T][n].  A hierarchical layer's dWg, dbg, dWn
        are the primary gate's, dWg2, dbg2, dWn2 the secondary gates'."""
        if not hasattr(self, "_grads"):
            cfg, dev = self.cfg, self.device
            z = lambda *shape: torch.zeros(*shape, dtype=torch.float32, device=dev)
            gn = cfg.hier_a if cfg.hier_a else cfg.n
            g = dict(dx=z(cfg.T, cfg.d), dWg=z(cfg.d, gn), dbg=z(gn),
                     dW1=z(cfg.n, cfg.f, cfg.d), db1=z(cfg.n, cfg.f), dW2=z(cfg.n, cfg.d, cfg.f),
                     db2=z(cfg.n, cfg.d))
            if cfg.noise:
                g["dWn"] = z(cfg.d, gn)
            if cfg.hier_a:
                g.update(dWg2=z(cfg.hier_a, cfg.d, cfg.hier_b), dbg2=z(cfg.hier_a, cfg.hier_b))
                if cfg.noise:
                    g["dWn2"] = z(cfg.hier_a, cfg.d, cfg.hier_b)
            if cfg.shared_expert:
                g.update(dW1s=z(cfg.f, cfg.d), db1s=z(cfg.f), dW2s=z(cfg.d, cfg.f), db2s=z(cfg.d))
            if intermediates:
                g["dgate"] = z(cfg.T, cfg.k)
                if not cfg.hier_a:
                    g["dlogits"] = z(cfg.T, cfg.n)
            self._grads = g
            self._mg = _lib.moe_grads(
                dW_g=_ptr(g["dWg"]), db_g=_ptr(g["dbg"]), dW_noise=_ptr(g.get("dWn")),
                dW1=_ptr(g["dW1"]), db1=_ptr(g["db1"]), dW2=_ptr(g["dW2"]), db2=_ptr(g["db2"]),
                dW1s=_ptr(g.get("dW1s")), db1s=_ptr(g.get("db1s")), dW2s=_ptr(g.get("dW2s")),
                db2s=_ptr(g.get("db2s")), dgate=_ptr(g.get("dgate")), dlogits=_ptr(g.get("dlogits")),
                dW_g2=_ptr(g.get("dWg2")), db_g2=_ptr(g.get("dbg2")), dW_noise2=_ptr(g.get("dWn2")))
        return self._grads

    def backward_(self, x: torch.Tensor, dy: torch.Tensor, stream=None,
                  dx: Optional[torch.Tensor] = None) -> dict:
        """Gradients of sum(dy * y) + the weighted balancing losses of the last
        forward_ (same x) into the buffers of grads() (dx into the given
        buffer when one is passed); asynchronous."""
        if not self.cfg.backward:
            raise MoEError("the layer was built without backward=1")
        _need(x, "x", torch.float32, (self.cfg.T, self.cfg.d), self.device)
        _need(dy, "dy", torch.float32, (self.cfg.T, self.cfg.d), self.device)
        g = self.grads()
        dx = g["dx"] if dx is None else dx
        _need(dx, "dx", torch.float32, (self.cfg.T, self.cfg.d), self.device)
        st = C.c_void_p(stream.cuda_stream) if stream is not None else _stream()
        _check(_lib.load().moe_backward(C.byref(self._c), _ptr(x), C.byref(self._gp),
                                        C.byref(self._ep), _ptr(dy), _ptr(self.topk_idx),
                                        _ptr(self.topk_gate), _ptr(self.importance),
                                        _ptr(self.load), _ptr(self.counts), _ptr(dx),
                                        C.byref(self._mg), _ptr(self.ws), self.ws.numel(),
                                        _ptr(self.status), st), "moe_backward")
        return g

    def train_host_batches(self, x_hosts, dy_hosts, y_hosts, losses_hosts, dx_hosts,
                           graph: bool = False):
        """Training steps (forward + backward) over batches in pinned host
        memory, pipelined like forward_host_batches: x and dy of batch i+1 go
        to the device and y, the losses and dx of batch i-1 come back on their
        own streams while batch i runs on the current stream (with graph each
        buffer set's step is replayed from a CUDA graph).  The parameter
        gradients stay on the device (those of the last batch).  Returns the
        device-to-host stream after queuing; the caller synchronises."""
        if not hasattr(self, "_tpipe"):
            dev = self.device
            e = lambda: [torch.empty_like(self.y) for _ in range(2)]
            self._tpipe = dict(h2d=torch.cuda.Stream(device=dev), d2h=torch.cuda.Stream(device=dev),
                               x=e(), dy=e(), y=e(), dx=e(),
                               losses=[torch.empty_like(self.losses) for _ in range(2)])
        P = self._tpipe
        comp = torch.cuda.current_stream(self.device)
        in_free = [None, None]    # event: device x / dy buffer b may be overwritten
        out_free = [None, None]   # event: device y / losses / dx buffer b has been copied out
        for i, (xh, dyh, yh, lh, dxh) in enumerate(zip(x_hosts, dy_hosts, y_hosts, losses_hosts,
                                                       dx_hosts)):
            b = i & 1
            with torch.cuda.stream(P["h2d"]):
                if in_free[b] is not None:
                    P["h2d"].wait_event(in_free[b])
                P["x"][b].copy_(xh, non_blocking=True)
                P["dy"][b].copy_(dyh, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(P["h2d"])
            comp.wait_event(ready)
            if out_free[b] is not None:
                comp.wait_event(out_free[b])
            if graph:
                self.train_graph_(P["x"][b], P["dy"][b], y=P["y"][b], losses=P["losses"][b],
                                  dx=P["dx"][b])
            else:
                self.forward_(P["x"][b], stream=comp, y=P["y"][b], losses=P["losses"][b])
                self.backward_(P["x"][b], P["dy"][b], stream=comp, dx=P["dx"][b])
            done = torch.cuda.Event()
            done.record(comp)
            in_free[b] = done
            with torch.cuda.stream(P["d2h"]):
                P["d2h"].wait_event(done)
                yh.copy_(P["y"][b], non_blocking=True)
                lh.copy_(P["losses"][b], non_blocking=True)
                dxh.copy_(P["dx"][b], non_blocking=True)
                out_free[b] = torch.cuda.Event()
                out_free[b].record(P["d2h"])
        return P["d2h"]

    def outputs(self) -> dict:
        return dict(y=self.y, topk_idx=self.topk_idx, topk_gate=self.topk_gate,
                    importance=self.importance, load=self.load, counts=self.counts,
                    losses=self.losses, status=self.status)

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, losses_host: torch.Tensor,
                     x_dev: torch.Tensor):
        """End-to-end call from host memory: copy x in (pinned host -> device),
        run the layer, copy y and the losses back, all on the current stream."""
        x_dev.copy_(x_host, non_blocking=True)
        self.forward_(x_dev)
        y_host.copy_(self.y, non_blocking=True)
        losses_host.copy_(self.losses, non_blocking=True)

    def forward_host_batches(self, x_hosts, y_hosts, losses_hosts, graph: bool = False):
        """End-to-end calls over a sequence of batches in pinned host memory,
        pipelined: the copy of batch i+1 to the device and the copy of batch
        i-1's y and losses to the host run on their own streams while batch i
        runs on the current stream (double-buffered device copies; with graph
        each buffer set's forward is replayed from a CUDA graph).  Returns
        after queuing; the caller synchronises."""
        if not hasattr(self, "_pipe"):
            dev = self.device
            self._pipe = dict(
                h2d=torch.cuda.Stream(device=dev), d2h=torch.cuda.Stream(device=dev),
                x=[torch.empty_like(self.y) for _ in range(2)],
                y=[torch.empty_like(self.y) for _ in range(2)],
                losses=[torch.empty_like(self.losses) for _ in range(2)])
        P = self._pipe
        comp = torch.cuda.current_stream(self.device)
        x_free = [None, None]   # event: device x buffer b may be overwritten
        y_free = [None, None]   # event: device y buffer b has been copied out
        for i, (xh, yh, lh) in enumerate(zip(x_hosts, y_hosts, losses_hosts)):
            b = i & 1
            with torch.cuda.stream(P["h2d"]):
                if x_free[b] is not None:
                    P["h2d"].wait_event(x_free[b])
                P["x"][b].copy_(xh, non_blocking=True)
                x_ready = torch.cuda.Event()
                x_ready.record(P["h2d"])
            comp.wait_event(x_ready)
            if y_free[b] is not None:
                comp.wait_event(y_free[b])
            if graph:
                self.forward_graph_(P["x"][b], y=P["y"][b], losses=P["losses"][b])
            else:
                self.forward_(P["x"][b], stream=comp, y=P["y"][b], losses=P["losses"][b])
            done = torch.cuda.Event()
            done.record(comp)
            x_free[b] = done
            with torch.cuda.stream(P["d2h"]):
                P["d2h"].wait_event(done)
                yh.copy_(P["y"][b], non_blocking=True)
                lh.copy_(P["losses"][b], non_blocking=True)
                y_free[b] = torch.cuda.Event()
                y_free[b].record(P["d2h"])
        return P["d2h"]


def forward(cfg: Config, x: torch.Tensor, params: dict) -> dict:
    layer = MoELayer(cfg, params, x.device)
    layer.forward_(x)
    return layer.outputs()


# ---------------------------------------------------------------- tracing
def sel_bias_update(cfg: Config, counts: torch.Tensor, gamma: float, sel_bias: torch.Tensor):
    """The sigmoid router's selection-bias update, in place on the current
    stream: experts with more than T*k/n of the slots in counts lose gamma,
    those with fewer gain it."""
    _need(counts, "counts", torch.int32, (cfg.n,), sel_bias.device)
    _need(sel_bias, "sel_bias", torch.float32, (cfg.n,), counts.device)
    c = cfg.c()
    _check(_lib.load().moe_sel_bias_update(C.byref(c), _ptr(counts), float(gamma), _ptr(sel_bias),
                                           _stream()), "moe_sel_bias_update")
    return sel_bias


def trace_enable(on: bool = True):
    _lib.load().moe_trace_enable(int(bool(on)))


def trace_reset():
    _lib.load().moe_trace_reset()


def trace_read() -> dict:
    L = _lib.load()
    out = {}
    for i in range(L.moe_trace_count()):
        name = C.c_char_p()
        nl = C.c_int()
        ms = C.c_double()
        _check(L.moe_trace_get(i, C.byref(name), C.byref(nl), C.byref(ms)), "moe_trace_get")
        out[name.value.decode()] = dict(launches=nl.value, ms=ms.value)
    return out


def launch_count() -> int:
    return int(_lib.load().moe_launch_count())
