"""B200 (sm_100a) forward pass of Kokoro's ALBERT phoneme encoder behind a C ABI.

The library ``libalbert_b200.so`` (built from ``csrc/`` by ``build.py``) does all
the work; this module only marshals arguments: it builds the C structs, passes
torch tensors' device pointers and the current CUDA stream, and turns non-zero
status codes into exceptions.  Nothing here computes any step of the encoder,
and there is no CPU fallback: if the library or a GPU is missing, calls fail.

The C functions are exposed under their own names (``albert_create``,
``albert_forward``, ``albert_forward_varlen``, ``albert_forward_host``,
``albert_get_status``, ``albert_destroy``) plus the ``Encoder`` convenience class.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libalbert_b200.so")

ALBERT_OK = 0
ALBERT_BF16, ALBERT_FP32, ALBERT_FP8 = 0, 1, 2
DTYPES = {"bf16": ALBERT_BF16, "fp32": ALBERT_FP32, "fp8": ALBERT_FP8}
STATUS_NAMES = {
    0: "ALBERT_OK", 1: "ALBERT_ERR_NULL", 2: "ALBERT_ERR_CONFIG", 3: "ALBERT_ERR_SHAPE",
    4: "ALBERT_ERR_ID", 5: "ALBERT_ERR_MASK", 6: "ALBERT_ERR_SEQLENS", 7: "ALBERT_ERR_CUDA",
    8: "ALBERT_ERR_TIMEOUT", 9: "ALBERT_ERR_ALLOC",
}

WEIGHT_FIELDS = (
    "word", "pos", "type", "emb_ln_g", "emb_ln_b", "w_in", "b_in",
    "wq", "bq", "wk", "bk", "wv", "bv", "wo", "bo", "ln1_g", "ln1_b",
    "w1", "b1", "w2", "b2", "ln2_g", "ln2_b", "w_out", "b_out",
)

EXPORTS = (
    "albert_create", "albert_forward", "albert_forward_varlen", "albert_forward_host",
    "albert_forward_host_async", "albert_forward_varlen_host_async", "albert_forward_host_wait",
    "albert_get_status", "albert_destroy", "albert_launches_per_forward",
    "albert_profile_enable", "albert_profile_retain", "albert_profile_stride", "albert_profile_reset",
    "albert_profile_classes",
    "albert_profile_name", "albert_profile_read", "albert_test_gemm", "albert_test_attention",
    "albert_gemm_residual_ln_noalloc", "albert_length_regulate", "albert_length_regulate_scratch_bytes",
    "albert_set_wait_limit", "albert_test_stall", "albert_set_small_batch_kernel", "albert_last_forward_launches",
    "albert_test_quant_e4m3", "albert_forward_embedded", "albert_test_attention_groups",
)


class AlbertError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


class albert_config(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("vocab", "emb", "hidden", "heads", "ffn", "n_exec", "n_groups",
                                       "max_pos", "n_types", "out_dim", "dtype", "max_tokens", "pack",
                                       "out_layout")] \
        + [("ln_eps", C.c_float)]


class albert_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in WEIGHT_FIELDS]


_lib = None


def lib() -> C.CDLL:
    """Load the CUDA library; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m transformer_encoder_albert_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i = C.c_void_p, C.c_int
        L.albert_create.argtypes = [C.POINTER(albert_weights), C.POINTER(albert_config), C.POINTER(vp)]
        L.albert_forward.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.albert_forward_varlen.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.albert_forward_host.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.albert_forward_host_async.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.albert_forward_varlen_host_async.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.albert_forward_host_wait.argtypes = [vp]
        L.albert_get_status.argtypes = [vp, vp]
        L.albert_destroy.argtypes = [vp]
        L.albert_destroy.restype = None
        L.albert_launches_per_forward.argtypes = [vp, i]
        L.albert_profile_enable.argtypes = [vp, i]
        L.albert_profile_reset.argtypes = [vp]
        L.albert_profile_retain.argtypes = [vp, i]
        L.albert_profile_stride.argtypes = [vp, i, i]
        L.albert_profile_classes.argtypes = []
        L.albert_profile_name.argtypes = [i]
        L.albert_profile_name.restype = C.c_char_p
        L.albert_profile_read.argtypes = [vp, C.POINTER(C.c_int), C.POINTER(C.c_double)]
        L.albert_test_gemm.argtypes = [vp, vp, vp, vp, vp, vp, C.c_float, vp, vp, i, i, i, i, vp]
        L.albert_test_attention.argtypes = [vp, vp, i, i, vp, i, vp]
        L.albert_gemm_residual_ln_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, C.c_float, vp, i, i, vp]
        L.albert_length_regulate.argtypes = [vp, i, C.c_float, vp, i, vp, i, i, vp, vp, vp, vp, i, vp, vp, vp]
        L.albert_length_regulate_scratch_bytes.argtypes = [i]
        L.albert_length_regulate_scratch_bytes.restype = C.c_size_t
        L.albert_set_wait_limit.argtypes = [vp, C.c_longlong]
        L.albert_test_stall.argtypes = [vp, i]
        L.albert_set_small_batch_kernel.argtypes = [vp, i]
        L.albert_last_forward_launches.argtypes = [vp]
        L.albert_test_quant_e4m3.argtypes = [vp, i, i, vp, vp, vp]
        L.albert_forward_embedded.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.albert_test_attention_groups.argtypes = [vp, i, i, vp, C.POINTER(C.c_int), vp]
        _lib = L
    return _lib


def _check(rc: int, where: str) -> None:
    if rc != ALBERT_OK:
        raise AlbertError(rc, where)


def _stream_ptr(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def make_config(arch: dict, dtype: str = "bf16", max_tokens: int = 4096, pack: bool = True,
                n_exec: int | None = None, out_dim: int | None = None, n_groups: int = 1,
                out_layout: int = 0) -> albert_config:
    return albert_config(
        vocab=arch["vocab"], emb=arch["emb"], hidden=arch["hidden"], heads=arch["heads"],
        ffn=arch["ffn"], n_exec=arch["n_exec"] if n_exec is None else n_exec, n_groups=n_groups,
        max_pos=arch["max_pos"], n_types=arch["n_types"],
        out_dim=arch["out_dim"] if out_dim is None else out_dim,
        dtype=DTYPES[dtype], max_tokens=max_tokens,
        pack=1 if pack else 0, out_layout=out_layout, ln_eps=arch["ln_eps"])


# ---------------------------------------------------------------- C names --

def albert_create(weights: dict, cfg: albert_config) -> int:
    """weights: name -> CUDA float32 tensor (contiguous).  Returns the handle."""
    import torch
    dev = {}
    for k in WEIGHT_FIELDS:
        t = weights.get(k)
        if t is None:
            dev[k] = None
            continue
        if not torch.is_tensor(t):
            t = torch.as_tensor(t)
        dev[k] = t.to(device="cuda", dtype=torch.float32).contiguous()
    w = albert_weights(*[_ptr(dev[k]) for k in WEIGHT_FIELDS])
    h = C.c_void_p()
    _check(lib().albert_create(C.byref(w), C.byref(cfg), C.byref(h)), "albert_create")
    return h.value


def albert_forward(h: int, ids, mask, out, stream=None) -> None:
    B, T = ids.shape
    _check(lib().albert_forward(h, _ptr(ids), _ptr(mask), B, T, _ptr(out), _stream_ptr(stream)),
           "albert_forward")


def albert_forward_varlen(h: int, ids, cu_seqlens, max_len: int, out, stream=None) -> None:
    nseq = cu_seqlens.numel() - 1
    _check(lib().albert_forward_varlen(h, _ptr(ids), _ptr(cu_seqlens), nseq, int(max_len), _ptr(out),
                                       _stream_ptr(stream)), "albert_forward_varlen")


def albert_forward_host(h: int, ids_host, mask_host, out_host, stream=None) -> int:
    B, T = ids_host.shape
    return lib().albert_forward_host(h, _ptr(ids_host), _ptr(mask_host), B, T, _ptr(out_host),
                                     _stream_ptr(stream))


def albert_forward_host_async(h: int, ids_host, mask_host, out_host, stream=None) -> int:
    B, T = ids_host.shape
    return lib().albert_forward_host_async(h, _ptr(ids_host), _ptr(mask_host), B, T, _ptr(out_host),
                                           _stream_ptr(stream))


def albert_forward_varlen_host_async(h: int, ids_host, cu_seqlens_host, max_len: int, out_host,
                                     stream=None) -> int:
    nseq = cu_seqlens_host.numel() - 1
    return lib().albert_forward_varlen_host_async(h, _ptr(ids_host), _ptr(cu_seqlens_host), nseq, int(max_len),
                                                  _ptr(out_host), _stream_ptr(stream))


def albert_forward_host_wait(h: int) -> int:
    return lib().albert_forward_host_wait(h)


def albert_get_status(h: int, stream=None) -> int:
    return lib().albert_get_status(h, _stream_ptr(stream))


def albert_destroy(h: int) -> None:
    lib().albert_destroy(h)


# --------------------------------------------------------- convenience class --

class Encoder:
    """Owns one library handle.  Outputs are bf16 (dtype "bf16") or fp32 tensors."""

    def __init__(self, weights: dict, arch: dict, dtype: str = "bf16", max_tokens: int = 4096,
                 pack: bool = True, n_exec: int | None = None, out_dim: int | None = None, n_groups: int = 1,
                 out_layout: int = 0):
        """n_groups > 1: the layer parameters of `weights` hold n_groups stacked sets
        (leading axis), execution i using set i * n_groups // n_exec.  out_layout 1:
        forward() returns [B, D, T] (each sequence's output transposed)."""
        self.cfg = make_config(arch, dtype, max_tokens, pack, n_exec, out_dim, n_groups, out_layout)
        self.out_layout = out_layout
        self.dtype = dtype
        self.out_dim = self.cfg.out_dim if self.cfg.out_dim > 0 else self.cfg.hidden
        self.h = albert_create(weights, self.cfg)

    def _out(self, shape):
        import torch
        dt = torch.float32 if self.dtype == "fp32" else torch.bfloat16
        return torch.empty(*shape, self.out_dim, device="cuda", dtype=dt)

    def forward(self, ids, mask, out=None, stream=None):
        if out is None:
            if self.out_layout == 1:
                import torch
                dt = torch.float32 if self.dtype == "fp32" else torch.bfloat16
                out = torch.empty(ids.shape[0], self.out_dim, ids.shape[1], device="cuda", dtype=dt)
            else:
                out = self._out(ids.shape)
        albert_forward(self.h, ids, mask, out, stream)
        return out

    def forward_varlen(self, ids, cu_seqlens, max_len, out=None, stream=None):
        if out is None:
            out = self._out((ids.shape[0],))
        albert_forward_varlen(self.h, ids, cu_seqlens, max_len, out, stream)
        return out

    def forward_embedded(self, emb, cu_seqlens, max_len, out=None, stream=None):
        """From post-embedding-LayerNorm rows emb [N_tok, 128] fp32 (packed as in
        forward_varlen) to the encoder output [N_tok, D]."""
        if out is None:
            out = self._out((emb.shape[0],))
        nseq = cu_seqlens.numel() - 1
        _check(lib().albert_forward_embedded(self.h, _ptr(emb), _ptr(cu_seqlens), nseq, int(max_len), _ptr(out),
                                             _stream_ptr(stream)), "albert_forward_embedded")
        return out

    def forward_host(self, ids_host, mask_host, out_host, stream=None) -> int:
        return albert_forward_host(self.h, ids_host, mask_host, out_host, stream)

    def forward_host_async(self, ids_host, mask_host, out_host, stream=None) -> int:
        """Enqueue one batch of the pipelined host path; returns the status of the
        batch issued two calls earlier (its output is then in host memory)."""
        return albert_forward_host_async(self.h, ids_host, mask_host, out_host, stream)

    def forward_varlen_host_async(self, ids_host, cu_seqlens_host, max_len: int, out_host, stream=None) -> int:
        """The pipelined host path for a packed batch: int64 ids [n_tok] and int32
        cu_seqlens [nseq + 1] in host memory, out_host [n_tok, out_dim]."""
        return albert_forward_varlen_host_async(self.h, ids_host, cu_seqlens_host, max_len, out_host, stream)

    def forward_host_wait(self) -> int:
        """Wait for all pipelined host batches; first non-OK status."""
        return albert_forward_host_wait(self.h)

    def status(self, stream=None) -> int:
        return albert_get_status(self.h, stream)

    def set_small_batch_kernel(self, enable: bool) -> None:
        """Batches of at most 128 token rows: one persistent kernel (True, default)
        or the per-layer kernels (False)."""
        _check(lib().albert_set_small_batch_kernel(self.h, 1 if enable else 0), "albert_set_small_batch_kernel")

    def last_forward_launches(self) -> int:
        return lib().albert_last_forward_launches(self.h)

    def set_wait_limit(self, ns: int) -> None:
        """Limit (ns) of the kernels' bounded waits on later forwards; 0 = default (2 s)."""
        _check(lib().albert_set_wait_limit(self.h, int(ns)), "albert_set_wait_limit")

    def test_stall(self, classes=()) -> None:
        """Failure injection: the GEMM launches of these kernel classes withhold
        their operand loads on later forwards, so their waits run out ([] = off)."""
        names = profile_class_names()
        mask = 0
        for c in classes:
            mask |= 1 << names.index(c)
        _check(lib().albert_test_stall(self.h, mask), "albert_test_stall")

    def launches_per_forward(self, padded_api: bool = True) -> int:
        return lib().albert_launches_per_forward(self.h, 1 if padded_api else 0)

    def profile(self, classes=None) -> None:
        """Time launches of the named kernel classes (None = all, [] = off)."""
        if classes is None:
            mask = -1
        else:
            names = profile_class_names()
            mask = 0
            for c in classes:
                mask |= 1 << names.index(c)
        _check(lib().albert_profile_enable(self.h, mask), "albert_profile_enable")

    def profile_retain(self, on: bool) -> None:
        """Keep recorded event pairs armed across reads (CUDA-graph replays)."""
        _check(lib().albert_profile_retain(self.h, 1 if on else 0), "albert_profile_retain")

    def profile_stride(self, stride: int, offset: int = 0) -> None:
        """Time only launch k of each enabled class with k % stride == offset."""
        _check(lib().albert_profile_stride(self.h, stride, offset), "albert_profile_stride")

    def profile_reset(self) -> None:
        _check(lib().albert_profile_reset(self.h), "albert_profile_reset")

    def profile_read(self) -> dict:
        n = lib().albert_profile_classes()
        launches = (C.c_int * n)()
        ms = (C.c_double * n)()
        _check(lib().albert_profile_read(self.h, launches, ms), "albert_profile_read")
        return {lib().albert_profile_name(i).decode(): (launches[i], ms[i]) for i in range(n)}

    def close(self) -> None:
        if self.h:
            albert_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def profile_class_names() -> list:
    n = lib().albert_profile_classes()
    return [lib().albert_profile_name(i).decode() for i in range(n)]


GEMM_VARIANTS = {"auto": 0, "single": 16, "pair": 32, "narrow": 128}
GEMM_E4M3 = 64


def test_gemm(A, W, bias, Y, epi: int, R=None, ln_g=None, ln_b=None, eps: float = 1e-12,
              row_dst=None, stream=None, variant: str = "auto", e4m3: bool = False) -> int:
    """Run the tcgen05 GEMM alone (single-kernel parity tests).  variant picks
    the one-CTA 128x256, the CTA-pair 256x256 or the one-CTA 128x128 kernel
    ("auto": the forward's choice); e4m3
    quantizes both operands per row and runs the E4M3 variant."""
    M, K = A.shape
    N = W.shape[0]
    return lib().albert_test_gemm(_ptr(A), _ptr(W), _ptr(bias), _ptr(R), _ptr(ln_g), _ptr(ln_b),
                                  float(eps), _ptr(row_dst), _ptr(Y), M, N, K,
                                  epi | GEMM_VARIANTS[variant] | (GEMM_E4M3 if e4m3 else 0), _stream_ptr(stream))


def test_attention_groups(cu_seqlens, max_len: int, stream=None):
    """The attention groups the forward forms for a packed batch: a list of
    (start row, length, partner start row, partner length (0: none))."""
    import numpy as np
    nseq = cu_seqlens.numel() - 1
    buf = np.zeros((nseq, 4), dtype=np.int32)
    n = C.c_int(0)
    _check(lib().albert_test_attention_groups(_ptr(cu_seqlens), nseq, int(max_len), buf.ctypes.data, C.byref(n),
                                              _stream_ptr(stream)), "albert_test_attention_groups")
    return [tuple(int(x) for x in g) for g in buf[:n.value]]


def test_quant_e4m3(x, stream=None):
    """Row quantization of the E4M3 variant: (codes [rows, K] uint8, scales [rows] fp32)."""
    import torch
    rows, K = x.shape
    q = torch.empty(rows, K, dtype=torch.uint8, device=x.device)
    s = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(lib().albert_test_quant_e4m3(_ptr(x), rows, K, _ptr(q), _ptr(s), _stream_ptr(stream)),
           "albert_test_quant_e4m3")
    return q, s


def test_attention(qkv, cu_seqlens, max_len: int, ctx, fp32: bool = False, legacy: bool = False,
                   stream=None) -> int:
    """Run the attention kernel alone (single-kernel parity tests); legacy forces
    the mma.sync kernel for bf16."""
    mode = ALBERT_FP32 if fp32 else (2 if legacy else ALBERT_BF16)
    return lib().albert_test_attention(_ptr(qkv), _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                                       int(max_len), _ptr(ctx), mode, _stream_ptr(stream))


def gemm_residual_ln_noalloc(A, W, bias, R, ln_g, ln_b, Y, eps: float = 1e-12, stream=None) -> int:
    """Y = LN(A W^T + bias + R) through the entry point that allocates no device
    memory (static scratch inside the library; M <= 2048).  The C side cannot see
    the tensors' extents, so they are checked here: a mismatched tensor would make
    the kernels read or write past the caller's buffers."""
    import torch
    M, K = A.shape
    N = 768
    want = {"A": (A, (M, K), torch.bfloat16), "W": (W, (N, K), torch.bfloat16), "R": (R, (M, N), torch.bfloat16),
            "Y": (Y, (M, N), torch.bfloat16), "bias": (bias, (N,), torch.float32),
            "ln_g": (ln_g, (N,), torch.float32), "ln_b": (ln_b, (N,), torch.float32)}
    for name, (t, shape, dt) in want.items():
        if tuple(t.shape) != shape or t.dtype != dt or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"gemm_residual_ln_noalloc: {name} must be a contiguous CUDA {dt} tensor "
                             f"of shape {shape}, got {tuple(t.shape)} {t.dtype} on {t.device}")
    return lib().albert_gemm_residual_ln_noalloc(_ptr(A), _ptr(W), _ptr(bias), _ptr(R), _ptr(ln_g),
                                                 _ptr(ln_b), float(eps), _ptr(Y), M, K,
                                                 _stream_ptr(stream))


def length_regulate(logits, feats, cu_seqlens, speed: float = 1.0, max_frames: int | None = None,
                    stream=None):
    """Length regulation of a packed batch on the GPU (albert_length_regulate).

    logits [n_tok, C] fp32, feats [n_tok, D] bf16, cu_seqlens [nseq+1] int32, all on
    the device.  Returns (status, durations, frame_start, cu_frames, frames) with
    frames [max_frames, D] (the first cu_frames[-1] rows hold the result)."""
    import torch
    n_tok, C = logits.shape
    D = feats.shape[1]
    nseq = cu_seqlens.numel() - 1
    if max_frames is None:
        max_frames = 64 * n_tok
    dev = logits.device
    dur = torch.empty(n_tok, dtype=torch.int32, device=dev)
    start = torch.empty(n_tok, dtype=torch.int32, device=dev)
    cu_frames = torch.empty(nseq + 1, dtype=torch.int32, device=dev)
    frames = torch.empty(max_frames, D, dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scratch = torch.empty(int(lib().albert_length_regulate_scratch_bytes(n_tok)), dtype=torch.uint8, device=dev)
    rc = lib().albert_length_regulate(_ptr(logits), C, float(speed), _ptr(feats), D, _ptr(cu_seqlens), nseq, n_tok,
                                      _ptr(dur), _ptr(start), _ptr(cu_frames), _ptr(frames), max_frames,
                                      _ptr(scratch), _ptr(status), _stream_ptr(stream))
    if rc != ALBERT_OK:
        return rc, None, None, None, None
    torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    return int(status.item()), dur, start, cu_frames, frames
