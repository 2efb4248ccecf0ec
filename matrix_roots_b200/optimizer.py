"""One blocked-Shampoo optimizer step as a sequence of the five C-ABI calls.

With ``precond_every`` = f > 1 the roots are recomputed only on steps 1,
1 + f, ... and the stale roots precondition the steps between ("3D-Shampoo
optimizer" README, Hyperparameters: preconditioning_compute_steps; DASH §1,
roots every 10-100 steps); the statistics are updated on steps 1,
1 + s, ... with ``stats_every`` = s (statistics_compute_steps; default
every step).
Method "evd" takes the roots from shampoo_inv_root_evd (blocks up to 128)
with the dampening heuristic ``evd_heuristic`` (DASH B.1-B.2).  Layers
listed in ``one_sided`` keep only left statistics and step along
L^(-1/2) G ("Shampoo" notes, "Roots on idle CPUs": embeddings, softmax and
layers too large for a right factor).  ``matrix_view`` gives the matrix an
N-d parameter is preconditioned as (DASH D: a (E, 3, 16, 16) patch
embedding becomes (E, 768)).

``BlockedShampoo`` owns the device state (gradient / factor / root /
direction stacks, graft moments and one shared workspace) and calls, in
order: shampoo_stack_blocks, shampoo_update_stats, shampoo_inv_root (once
per factor bucket), shampoo_precondition and shampoo_graft_step.  Every
arithmetic step runs in the library's CUDA kernels; this module only
allocates tensors and marshals arguments.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import binding as B
from . import workloads


def matrix_shape(shape):
    """(first dimension, product of the rest) for rank >= 2; None for rank
    0 and 1 (left to a diagonal optimizer)."""
    shape = tuple(int(x) for x in shape)
    if len(shape) < 2:
        return None
    rest = 1
    for x in shape[1:]:
        rest *= x
    return (shape[0], rest)


def matrix_view(t):
    """The 2-D view of a contiguous parameter or gradient tensor that the
    optimizer preconditions (``matrix_shape``); None for vectors."""
    shp = matrix_shape(t.shape)
    return None if shp is None else t.view(shp)


@dataclass
class ShampooConfig:
    block_size: int = 1024
    beta2: float = 1.0          # statistics decay
    alpha: float = 1.0          # statistics weight (1 - beta2 for a moving average)
    eps: float = 1e-6
    method: str = "ndb"
    iters: int = 20             # iterations per call, or the Chebyshev degree
    dtype: str = "fp32"         # root iterations
    stats_dtype: str = "fp32"
    precond_dtype: str = "fp32"
    scaling: str = "frobenius"
    pi_vectors: int = 16
    pi_iters: int = 10
    pi_seed: int = 0
    graft: str = "sgd"
    lr: float = 0.1
    beta1: float = 0.9
    graft_beta2: float = 0.999
    graft_eps: float = 1e-8
    weight_decay: float = 0.0
    graft_per_block: bool = False
    precond_every: int = 1      # roots on steps 1, 1+f, 1+2f, ...
    stats_every: int = 1        # statistics on steps 1, 1+s, 1+2s, ...
    root_p: int = 4             # inverse p-th roots, p in (2, 4, 8)
    graph: bool = False         # replay the launches before the graft step as a CUDA graph
    layerwise: bool = False     # stack per layer instead of across all layers
    evd_heuristic: str = "corrected"  # method "evd": corrected, shifted_relu, abs_add or shmp
    one_sided: tuple = ()       # layer indices preconditioned on the left only, D = L^(-1/2) G

    def check(self, n_layers: int | None = None) -> None:
        """Raises ValueError for an option the library would refuse or
        misread; run before any device memory is allocated."""
        def one_of(name, value, allowed):
            if value not in allowed:
                raise ValueError(f"{name} must be one of {sorted(allowed)}, not {value!r}")
        one_of("method", self.method, set(B.METHODS) | {"evd"})
        for name in ("dtype", "stats_dtype", "precond_dtype"):
            one_of(name, getattr(self, name), set(B.DTYPES))
        one_of("scaling", self.scaling, set(B.SCALINGS))
        one_of("graft", self.graft, set(B.GRAFTS))
        one_of("evd_heuristic", self.evd_heuristic, set(B.EVD_HEURISTICS))
        one_of("root_p", self.root_p, {2, 4, 8})
        if self.block_size < 0:
            raise ValueError("block_size must be >= 0 (0: no blocking)")
        if self.precond_every < 1 or self.stats_every < 1:
            raise ValueError("precond_every and stats_every must be >= 1")
        if self.method != "evd" and not (1 <= self.iters <= 1000 or (self.method == "cheb" and self.iters == 0)):
            raise ValueError("iters must be in [1, 1000] (a Chebyshev degree may be 0)")
        if not (self.eps >= 0.0) or self.eps == float("inf"):
            raise ValueError("eps must be finite and >= 0")
        if self.scaling == "power" and (self.pi_vectors < 8 or self.pi_vectors > 256 or self.pi_vectors % 8):
            raise ValueError("pi_vectors must be a multiple of 8 in [8, 256]")
        if self.method == "evd" and 0 < self.block_size and self.block_size > B.EVD_MAX_N:
            raise ValueError(f"method 'evd' needs blocks of at most {B.EVD_MAX_N} (block_size {self.block_size})")
        if n_layers is not None and any(not 0 <= i < n_layers for i in self.one_sided):
            raise ValueError(f"one_sided indices must name layers 0..{n_layers - 1}")


class BlockedShampoo:
    def __init__(self, shapes, cfg: ShampooConfig, device="cuda"):
        import torch
        cfg.check(len(shapes))
        self.cfg = cfg
        self.device = torch.device(device)
        self.shapes = [(int(m), int(n)) for m, n in shapes]
        left_only = [i in set(cfg.one_sided) for i in range(len(self.shapes))] if cfg.one_sided else None
        self.plan = B.Plan(self.shapes, cfg.block_size, cfg.layerwise, left_only).bind(self.device)
        t = self.plan.tables()
        self.tables = t
        f32 = dict(dtype=torch.float32, device=self.device)
        self.g_stacks = [torch.empty((int(c), int(r), int(k)), **f32) for r, k, c in t["g_buckets"]]
        self.d_stacks = [torch.empty_like(g) for g in self.g_stacks]
        self.factors = [torch.zeros((int(c), int(n), int(n)), **f32) for n, c in t["f_buckets"]]
        self.roots = [torch.empty_like(f) for f in self.factors]
        self.scales = [torch.empty(int(c), **f32) for _, c in t["f_buckets"]]
        self.status = [torch.empty(int(c), dtype=torch.int32, device=self.device) for _, c in t["f_buckets"]]
        self.dnorm2 = torch.empty(self.plan.n_blocks, **f32)
        self.m = [torch.zeros(s, **f32) for s in self.shapes] if cfg.graft == "adam" else None
        self.v = [torch.zeros(s, **f32) for s in self.shapes] if cfg.graft in ("adam", "adagrad") else None
        self.pi_starts = {}
        if cfg.scaling == "power":
            for n, _ in t["f_buckets"]:
                s = workloads.power_iteration_starts(int(n), cfg.pi_vectors, cfg.pi_seed)
                self.pi_starts[int(n)] = torch.from_numpy(s).to(self.device)
        need = max(
            [B.update_stats_workspace_bytes(self.plan, cfg.stats_dtype),
             B.precondition_workspace_bytes(self.plan, cfg.precond_dtype),
             B.graft_step_workspace_bytes(self.plan)]
            + [B.inv_root_workspace_bytes(int(c), int(n), cfg.method, cfg.dtype, cfg.scaling, cfg.pi_vectors)
               for n, c in (t["f_buckets"] if cfg.method != "evd" else [])])
        self.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        self.t = 0
        self._graphs = {}       # (fresh roots?, gradient addresses) -> (CUDAGraph, library launches in it)
        self.graph_launches = 0  # library kernel launches replayed from graphs so far

    def state_dict(self) -> dict:
        """The optimizer state as host tensors -- step count, statistics,
        the current roots (reused until the next refresh), graft moments --
        so that a run can be checkpointed and resumed; the weights stay with
        the caller."""
        def host(ts):
            return None if ts is None else [t.detach().to("cpu", copy=True) for t in ts]
        return {"t": self.t, "shapes": [list(s) for s in self.shapes], "factors": host(self.factors),
                "roots": host(self.roots), "m": host(self.m), "v": host(self.v)}

    def load_state_dict(self, state: dict) -> None:
        """Restores ``state_dict()`` output of an optimizer with the same
        shapes and configuration (copied into the existing device tensors, so
        captured CUDA graphs stay valid)."""
        if [tuple(int(x) for x in s) for s in state["shapes"]] != self.shapes:
            raise ValueError("state was saved for other layer shapes")
        for name in ("factors", "roots", "m", "v"):
            dst, src = getattr(self, name), state[name]
            if (dst is None) != (src is None) or (dst is not None and len(dst) != len(src)):
                raise ValueError(f"state entry {name!r} does not match this optimizer's configuration")
            for d, x in zip(dst or [], src or []):
                if tuple(d.shape) != tuple(x.shape):
                    raise ValueError(f"state entry {name!r} has shape {tuple(x.shape)}, expected {tuple(d.shape)}")
                d.copy_(x)
        self.t = int(state["t"])

    def _direction(self, G, stream, fresh: bool, stats: bool = True) -> None:
        """Stack, statistics (when ``stats``), roots (when fresh) and D for
        gradients G."""
        c = self.cfg
        ws = self.workspace
        B.stack_blocks(self.plan, G, self.g_stacks, stream)
        if stats:
            B.update_stats(self.plan, self.g_stacks, self.factors, c.beta2, c.alpha, c.stats_dtype, ws, stream)
        for fb, (n, _) in enumerate(self.tables["f_buckets"] if fresh else []):
            p = 2 if self.tables["f_sides"][fb] else c.root_p  # one-sided layers: L^(-1/2)
            if c.method == "evd":
                B.inv_root_evd(self.factors[fb], c.eps, c.evd_heuristic, p, out=self.roots[fb],
                               status_out=self.status[fb], stream=stream)
                continue
            B.inv_root(self.factors[fb], c.eps, c.method, c.iters, c.dtype, c.scaling, p, c.pi_vectors, c.pi_iters,
                       self.pi_starts.get(int(n)), self.roots[fb], self.scales[fb], self.status[fb], ws, stream)
        B.precondition(self.plan, self.roots, self.g_stacks, self.d_stacks, self.dnorm2, c.precond_dtype, ws,
                       stream)

    def _direction_graphed(self, G, fresh: bool, stats: bool = True) -> None:
        """The same launches replayed from a CUDA graph captured on the first
        step that sees these gradient tensors (their addresses are part of
        the graph: refill the same tensors every step).  The first such step
        runs eagerly, so every kernel is set up before the capture."""
        import torch
        key = (fresh, stats, tuple(int(g.data_ptr()) for g in G))
        if key not in self._graphs:
            if (None,) + key not in self._graphs:
                self._graphs[(None,) + key] = None  # seen once: run eagerly
                self._direction(G, None, fresh, stats)
                return
            graph = torch.cuda.CUDAGraph()
            before = B.launch_count()
            torch.cuda.synchronize(self.device)
            with torch.cuda.graph(graph):
                self._direction(G, None, fresh, stats)
            self._graphs[key] = (graph, B.launch_count() - before)
        graph, n = self._graphs[key]
        graph.replay()
        self.graph_launches += n

    def step(self, W, G, stream=None) -> None:
        """W <- W - lr * rho * D - lr * wd * W for every layer, in place.  With
        ``graph`` the work before the graft step replays as a CUDA graph on the
        current stream (the graft step's bias corrections change every step,
        so it always launches directly)."""
        c = self.cfg
        ws = self.workspace
        self.t += 1
        fresh = (self.t - 1) % max(int(c.precond_every), 1) == 0
        stats = (self.t - 1) % max(int(c.stats_every), 1) == 0
        if c.graph:
            self._direction_graphed(G, fresh, stats)
        else:
            self._direction(G, stream, fresh, stats)
        B.graft_step(self.plan, W, G, self.d_stacks, self.dnorm2, self.m, self.v, c.graft, c.lr, c.beta1,
                     c.graft_beta2, c.graft_eps, c.weight_decay, self.t, c.graft_per_block, ws, stream)
