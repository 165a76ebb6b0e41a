"""PyTorch-facing wrapper over the C ABI.

PyTorch supplies device memory (the caller's tensors and the two workspaces)
and the CUDA stream; every step of the computation runs in the native
library. Nothing here computes on tensor values.
"""
import ctypes

import numpy as np
import torch

from . import _native as N


def make_policy(kind, block=128, tile=(1, 1, 128), topk=0, keep_diagonal=False,
                window=(1, 1, 1), temporal_heads=None, heads=0, sink_tokens=0, frame_radius=1,
                candidates=(), top_p=0.0, fg_group=64, fg_keep_fraction=0.15,
                explicit_layout=N.SA_LAYOUT_IDENTITY, explicit_bits=None, summarizer="mean",
                head_windows=None):
    """Fill an ``sa_policy``. ``kind`` is a name ("topk", "sta", "spatiotemporal",
    "spade", "fg", "explicit") or an SA_MASK_* code; ``summarizer`` ("mean",
    "max", "min" or an SA_SUMMARIZER_* code) picks the block summary behind the
    pooled scores of "topk" and "spade"; ``head_windows`` (one odd (wt, wh, ww)
    per head) gives "sta" a window per head."""
    names = {"topk": N.SA_MASK_TOPK, "sta": N.SA_MASK_STA,
             "spatiotemporal": N.SA_MASK_SPATIOTEMPORAL, "spade": N.SA_MASK_SPADE,
             "fg": N.SA_MASK_FG, "explicit": N.SA_MASK_EXPLICIT}
    p = N.Policy()
    p.kind = names.get(kind, kind)
    p.block = block
    p.tile[:] = list(tile)
    p.topk = topk
    p.keep_diagonal = 1 if keep_diagonal else 0
    p.window[:] = list(window)
    if temporal_heads is not None:
        arr = (ctypes.c_int8 * max(1, heads))()
        for h in temporal_heads:
            if not 0 <= h < heads:
                raise ValueError(f"temporal head {h} is outside 0..{heads - 1} (pass heads=)")
            arr[h] = 1
        p.head_is_temporal = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int8))
        p._keep_alive = arr
    p.sink_tokens = sink_tokens
    p.frame_radius = frame_radius
    p.n_candidates = len(candidates)
    for i, c in enumerate(candidates):
        p.candidates[i][:] = list(c)
    p.top_p = top_p
    p.fg_group = fg_group
    p.fg_keep_fraction = fg_keep_fraction
    p.explicit_layout = explicit_layout
    sums = {"mean": N.SA_SUMMARIZER_MEAN, "max": N.SA_SUMMARIZER_MAX, "min": N.SA_SUMMARIZER_MIN}
    p.summarizer = sums.get(summarizer, summarizer)
    if head_windows is not None:
        if any(len(w) != 3 for w in head_windows):
            raise ValueError("each head window is (wt, wh, ww)")
        arr = (ctypes.c_int * (3 * len(head_windows)))(*[int(x) for w in head_windows for x in w])
        p.head_windows = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int))
        p._keep_windows = arr
    if explicit_bits is not None:
        p.explicit_bits = explicit_bits.data_ptr()
        p._keep_bits = explicit_bits
    return p


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_tensor(t, shape, dtypes, name, device=None):
    """Raise unless ``t`` is a contiguous CUDA tensor of one of ``dtypes`` and
    the given shape, on ``device`` when one is given. The kernels see only a
    pointer, so a wrong size here would read or write past the buffer."""
    ok = (isinstance(t, torch.Tensor) and t.dtype in dtypes and t.is_cuda and t.is_contiguous()
          and tuple(t.shape) == tuple(shape) and (device is None or t.device == device))
    if not ok:
        kinds = "/".join(str(d).replace("torch.", "") for d in dtypes)
        where = f" on {device}" if device is not None else ""
        got = (f"{t.dtype} {tuple(t.shape)} on {t.device}" if isinstance(t, torch.Tensor)
               else type(t).__name__)
        raise ValueError(f"{name} must be a contiguous CUDA {kinds} tensor of shape "
                         f"{tuple(shape)}{where}, got {got}")


def _qkv_shape(problem):
    return (problem.batch, problem.heads, problem.T * problem.H * problem.W, problem.head_dim)


def _check_qkv(t, problem, name, device=None):
    _check_tensor(t, _qkv_shape(problem), (torch.bfloat16,), name, device)


def _check_lse(t, problem, device):
    _check_tensor(t, _qkv_shape(problem)[:3], (torch.float32,), "lse", device)


def _check_host(t, shape, dtype, name):
    """Raise unless ``t`` is a contiguous CPU tensor of ``dtype`` and the given
    shape (the library copies exactly that many bytes from or to it)."""
    ok = (isinstance(t, torch.Tensor) and t.dtype == dtype and t.device.type == "cpu"
          and t.is_contiguous() and tuple(t.shape) == tuple(shape))
    if not ok:
        got = (f"{t.dtype} {tuple(t.shape)} on {t.device}" if isinstance(t, torch.Tensor)
               else type(t).__name__)
        raise ValueError(f"{name} must be a contiguous host {dtype} tensor of shape "
                         f"{tuple(shape)}, got {got}")


def _check_head_arrays(policy, heads):
    """The library reads one entry per head of the problem from the policy's
    host arrays; a policy made for fewer heads would be read past its end."""
    arr = getattr(policy, "_keep_alive", None)
    if policy.head_is_temporal and (arr is None or len(arr) < heads):
        raise ValueError(f"the policy's temporal-head flags cover "
                         f"{0 if arr is None else len(arr)} heads, the problem has {heads}")
    win = getattr(policy, "_keep_windows", None)
    if policy.head_windows and (win is None or len(win) < 3 * heads):
        raise ValueError(f"the policy's head_windows cover "
                         f"{0 if win is None else len(win) // 3} heads, the problem has {heads}")


def _check_scratch(ws, device):
    if not (isinstance(ws, torch.Tensor) and ws.is_cuda and ws.device == device
            and ws.is_contiguous() and ws.numel() * ws.element_size() >= 256):
        raise ValueError(f"scratch_ws must be a contiguous CUDA tensor of at least 256 bytes on {device}")


class SparseAttention:
    """Caller-owned workspaces plus the build-mask / forward calls for one problem."""

    def __init__(self, batch, heads, T, H, W, head_dim, policy, device="cuda"):
        self.problem = N.Problem(batch, heads, T, H, W, head_dim)
        self.policy = policy
        _check_head_arrays(policy, heads)
        self.mask_bytes, self.scratch_bytes = N.workspace_size(self.problem, policy)
        self.mask_ws = torch.empty(self.mask_bytes, dtype=torch.uint8, device=torch.device(device))
        self.device = self.mask_ws.device                 # "cuda" resolved to its index
        self.scratch_ws = torch.empty(max(self.scratch_bytes, 256), dtype=torch.uint8,
                                      device=self.device)
        if policy.kind == N.SA_MASK_EXPLICIT:
            self._check_explicit_bits()

    def _check_explicit_bits(self):
        bits = getattr(self.policy, "_keep_bits", None)
        if bits is None or not self.policy.explicit_bits:
            raise ValueError("an explicit policy needs explicit_bits")
        need = N.export_bytes(self.problem, self.policy, N.SA_EXPORT_BLOCK_BITS)
        if not (bits.is_cuda and bits.device == self.device and bits.is_contiguous()
                and bits.element_size() == 4 and not bits.is_floating_point()
                and bits.numel() * 4 == need):
            raise ValueError(f"explicit_bits must be a contiguous CUDA int32/uint32 tensor of "
                             f"{need // 4} words ([batch*heads][nb][ceil(nb/32)]) on {self.device}")

    @property
    def n_tokens(self):
        return self.problem.T * self.problem.H * self.problem.W

    def build_mask(self, q, k, stream=None):
        needs = self.policy.kind in (N.SA_MASK_TOPK, N.SA_MASK_SPADE, N.SA_MASK_FG)
        if needs:
            _check_qkv(q, self.problem, "q", self.device)
            _check_qkv(k, self.problem, "k", self.device)
        N.build_mask(self.problem, self.policy, q.data_ptr() if needs else None,
                     k.data_ptr() if needs else None, self.mask_ws.data_ptr(),
                     self.scratch_ws.data_ptr(), _stream_ptr(stream))

    def build_mask_fg_cached(self, q, k, lse, tau=0.0, stream=None):
        """FG cached mask (FG-Attn review, the cached strategy): slices that
        some query of their group gives a probability above ``tau`` (0: 0.5/N),
        from ``lse``, the float32 [batch, heads, N] LSE of full attention of q
        over all keys. The policy must be "fg"; its keep fraction only bounds
        the size of the union lists."""
        if self.policy.kind != N.SA_MASK_FG:
            raise ValueError("build_mask_fg_cached needs an \"fg\" policy")
        _check_qkv(q, self.problem, "q", self.device)
        _check_qkv(k, self.problem, "k", self.device)
        _check_lse(lse, self.problem, self.device)
        N.build_mask_fg_cached(self.problem, self.policy, q.data_ptr(), k.data_ptr(),
                               lse.data_ptr(), tau, self.mask_ws.data_ptr(),
                               self.scratch_ws.data_ptr(), _stream_ptr(stream))

    def forward(self, q, k, v, out=None, lse=None, stream=None):
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _check_qkv(t, self.problem, n, self.device)
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        _check_qkv(out, self.problem, "out", self.device)
        _check_lse(lse, self.problem, self.device)
        N.forward(self.problem, self.policy, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                  self.mask_ws.data_ptr(), self.scratch_ws.data_ptr(), out.data_ptr(),
                  lse.data_ptr(), _stream_ptr(stream))
        return out, lse

    def forward_host(self, q, k, v, out, lse=None, stream=None):
        """Build the mask and run the forward pass on host tensors: Q, K, V
        are copied in, O (and LSE when given) copied back, all queued on
        ``stream`` through one library call (sparse_attn_forward_host). The
        device staging buffers belong to this object, so calls of one object
        are ordered by their stream; page-locked host tensors keep the copies
        asynchronous."""
        shape = _qkv_shape(self.problem)
        for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
            _check_host(t, shape, torch.bfloat16, n)
        if lse is not None:
            _check_host(lse, shape[:3], torch.float32, "lse")
        if getattr(self, "_stage", None) is None:
            n = 1
            for s in shape:
                n *= s
            self._stage = (torch.empty(3 * n, dtype=torch.bfloat16, device=self.device),
                           torch.empty(n, dtype=torch.bfloat16, device=self.device),
                           torch.empty(shape[:3], dtype=torch.float32, device=self.device))
        qkv_d, o_d, lse_d = self._stage
        N.forward_host(self.problem, self.policy, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                       out.data_ptr(), lse.data_ptr() if lse is not None else None,
                       qkv_d.data_ptr(), o_d.data_ptr(),
                       lse_d.data_ptr() if lse is not None else None,
                       self.mask_ws.data_ptr(), self.scratch_ws.data_ptr(), _stream_ptr(stream))
        return out, lse

    def permute(self, q, k, v, stream=None):
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _check_qkv(t, self.problem, n, self.device)
        N.permute(self.problem, self.policy, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                  self.mask_ws.data_ptr(), self.scratch_ws.data_ptr(), _stream_ptr(stream))

    def attend(self, q, k, v, out, lse, stream=None):
        for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
            _check_qkv(t, self.problem, n, self.device)
        if lse is not None:
            _check_lse(lse, self.problem, self.device)
        N.attend(self.problem, self.policy, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                 self.mask_ws.data_ptr(), self.scratch_ws.data_ptr(), out.data_ptr(),
                 lse.data_ptr() if lse is not None else None, _stream_ptr(stream))
        return out, lse

    def forward_fp8(self, q, k, v, out=None, lse=None, stream=None):
        """FP8 attention over the built mask: Q, K and V quantized to E4M3 with
        one scale per (batch, head) tensor, frame-major copies of the codes,
        then the block-sparse attention on kind::f8f6f4 tensor cores. Returns
        (out, lse, (codes, inv) of q, k, v)."""
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _check_qkv(t, self.problem, n, self.device)
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        _check_qkv(out, self.problem, "out", self.device)
        _check_lse(lse, self.problem, self.device)
        quant = [quantize_e4m3(t, stream) for t in (q, k, v)]
        (q8, qi), (k8, ki), (v8, vi) = quant
        N.permute_fp8(self.problem, self.policy, q8.data_ptr(), k8.data_ptr(), v8.data_ptr(),
                      self.mask_ws.data_ptr(), self.scratch_ws.data_ptr(), _stream_ptr(stream))
        N.attend_fp8(self.problem, self.policy, q8.data_ptr(), k8.data_ptr(), v8.data_ptr(),
                     qi.data_ptr(), ki.data_ptr(), vi.data_ptr(), self.mask_ws.data_ptr(),
                     self.scratch_ws.data_ptr(), out.data_ptr(), lse.data_ptr(),
                     _stream_ptr(stream))
        return out, lse, quant

    def attend_fp8(self, q8, k8, v8, q_inv, k_inv, v_inv, out, lse, stream=None):
        """The FP8 attention step alone on existing codes and scales (after
        permute_fp8)."""
        N.attend_fp8(self.problem, self.policy, q8.data_ptr(), k8.data_ptr(), v8.data_ptr(),
                     q_inv.data_ptr(), k_inv.data_ptr(), v_inv.data_ptr(), self.mask_ws.data_ptr(),
                     self.scratch_ws.data_ptr(), out.data_ptr(), lse.data_ptr(),
                     _stream_ptr(stream))
        return out, lse

    def permute_fp8(self, q8, k8, v8, stream=None):
        N.permute_fp8(self.problem, self.policy, q8.data_ptr(), k8.data_ptr(), v8.data_ptr(),
                      self.mask_ws.data_ptr(), self.scratch_ws.data_ptr(), _stream_ptr(stream))

    def __call__(self, q, k, v, stream=None):
        self.build_mask(q, k, stream)
        return self.forward(q, k, v, stream=stream)

    def export(self, what, stream=None):
        nbytes = N.export_bytes(self.problem, self.policy, what)
        if what == N.SA_EXPORT_HEAD_INFO:
            buf = (N.HeadInfo * (nbytes // ctypes.sizeof(N.HeadInfo)))()
            N.mask_export(self.problem, self.policy, self.mask_ws.data_ptr(), what,
                          ctypes.addressof(buf), nbytes, _stream_ptr(stream))
            return list(buf)
        dtype = np.float32 if what == N.SA_EXPORT_FG_TAU else np.uint32
        arr = np.empty(nbytes // 4, dtype=dtype)
        N.mask_export(self.problem, self.policy, self.mask_ws.data_ptr(), what,
                      arr.ctypes.data, nbytes, _stream_ptr(stream))
        return arr

    def status(self, clear=False, stream=None):
        return N.status(self.scratch_ws.data_ptr(), _stream_ptr(stream), clear)


def _sampled_scratch(problem, n_rows, scratch_ws, device):
    """The scratch workspace of a sampled-row call: the caller's, checked for
    size, or a new one of sparse_attn_profile_workspace_size bytes."""
    need = N.profile_workspace_size(problem, n_rows)
    if scratch_ws is None:
        return torch.empty(need, dtype=torch.uint8, device=device)
    if scratch_ws.numel() * scratch_ws.element_size() < need:
        raise ValueError(f"scratch_ws holds {scratch_ws.numel() * scratch_ws.element_size()} "
                         f"bytes, the call needs {need}")
    return scratch_ws


def _sampled_problem(q, k, v, rows, T, H, W, scratch_ws):
    """Problem of a sampled-row call, after checking every tensor it is given."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a CUDA bf16 tensor [batch, heads, N, head_dim]")
    B, Hh, _, d = q.shape
    problem = N.Problem(B, Hh, T, H, W, d)
    if not (isinstance(rows, torch.Tensor) and rows.dim() == 2 and rows.shape[0] == B * Hh):
        raise ValueError("rows must be a contiguous CUDA int32 tensor [batch*heads, n_rows]")
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _check_qkv(t, problem, name, q.device)
    _check_tensor(rows, tuple(rows.shape), (torch.int32,), "rows", q.device)
    if scratch_ws is not None:
        _check_scratch(scratch_ws, q.device)
    return problem


def profile_heads(q, k, v, rows, T, H, W, block=128, sink_tokens=0, frame_radius=1,
                  stream=None, scratch_ws=None):
    """SVG online head profiler (Sparse VideoGen review, key machinery).

    q, k, v: contiguous CUDA bf16 [batch, heads, N, d]; rows: CUDA int32
    [batch*heads, n_rows] sampled query tokens. Returns (is_temporal int8
    [batch*heads], mse float32 [batch*heads, 2], row_err float32
    [batch*heads, n_rows, 2]) as CUDA tensors; the work is queued on
    ``stream`` and nothing is synchronised. ``scratch_ws`` (optional here)
    is the call's workspace; one of sparse_attn_profile_workspace_size bytes
    is made when it is None.
    """
    problem = _sampled_problem(q, k, v, rows, T, H, W, scratch_ws)
    B, Hh = problem.batch, problem.heads
    n_rows = rows.shape[1]
    policy = make_policy("spatiotemporal", block=block, temporal_heads=(), heads=Hh,
                         sink_tokens=sink_tokens, frame_radius=frame_radius)
    dev = q.device
    row_err = torch.empty((B * Hh, n_rows, 2), dtype=torch.float32, device=dev)
    mse = torch.empty((B * Hh, 2), dtype=torch.float32, device=dev)
    is_temporal = torch.empty(B * Hh, dtype=torch.int8, device=dev)
    scratch_ws = _sampled_scratch(problem, n_rows, scratch_ws, dev)
    N.profile_heads(problem, policy, q.data_ptr(), k.data_ptr(), v.data_ptr(), rows.data_ptr(),
                    n_rows, row_err.data_ptr(), mse.data_ptr(), is_temporal.data_ptr(),
                    scratch_ws.data_ptr(), _stream_ptr(stream))
    return is_temporal, mse, row_err


def sta_window_search(q, k, v, rows, T, H, W, tile, candidates, block=128, stream=None,
                      scratch_ws=None):
    """STA per-head window search (Sliding Tile Attention review, key machinery).

    q, k, v: contiguous CUDA bf16 [batch, heads, N, d]; rows: CUDA int32
    [batch*heads, n_rows]; tile: (bt, bh, bw) with bt*bh*bw == block;
    candidates: odd (wt, wh, ww) windows in tiles. Returns (choice int8
    [batch*heads], mse float32 [batch*heads, n_candidates], row_err float32
    [batch*heads, n_rows, n_candidates]) as CUDA tensors, queued on ``stream``.
    ``[candidates[c] for c in choice]`` is a ``head_windows`` for make_policy.
    """
    problem = _sampled_problem(q, k, v, rows, T, H, W, scratch_ws)
    B, Hh = problem.batch, problem.heads
    n_rows, nc = rows.shape[1], len(candidates)
    policy = make_policy("sta", block=block, tile=tile, window=(1, 1, 1))
    cand = (ctypes.c_int * (3 * nc))(*[int(x) for c in candidates for x in c])
    dev = q.device
    row_err = torch.empty((B * Hh, n_rows, nc), dtype=torch.float32, device=dev)
    mse = torch.empty((B * Hh, nc), dtype=torch.float32, device=dev)
    choice = torch.empty(B * Hh, dtype=torch.int8, device=dev)
    scratch_ws = _sampled_scratch(problem, n_rows, scratch_ws, dev)
    N.sta_window_search(problem, policy, q.data_ptr(), k.data_ptr(), v.data_ptr(), rows.data_ptr(),
                        n_rows, cand, nc, row_err.data_ptr(), mse.data_ptr(), choice.data_ptr(),
                        scratch_ws.data_ptr(), _stream_ptr(stream))
    return choice, mse, row_err



def quantize_e4m3(x, stream=None):
    """E4M3 codes of a contiguous CUDA bf16 tensor [batch, heads, N, d] with one
    scale per (batch, head) (Sparse VideoGen review: FP8 quantization).
    Returns (codes uint8, same shape; inv float32 [batch*heads]), queued on
    ``stream``; the dequantized operand is codes' value / inv."""
    if not (isinstance(x, torch.Tensor) and x.dim() == 4):
        raise ValueError("x must be a CUDA bf16 tensor [batch, heads, N, head_dim]")
    _check_tensor(x, tuple(x.shape), (torch.bfloat16,), "x")
    n_tensors = x.shape[0] * x.shape[1]
    n_elems = x.shape[2] * x.shape[3]
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    inv = torch.empty(n_tensors, dtype=torch.float32, device=x.device)
    N.quantize_e4m3(x.data_ptr(), n_elems, n_tensors, codes.data_ptr(), inv.data_ptr(),
                    _stream_ptr(stream))
    return codes, inv
