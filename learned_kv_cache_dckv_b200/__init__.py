"""B200-native DCKV codec: Python binding of the C ABI in include/dckv.h.

The binding only marshals arguments: every step of encode and decode runs in the
CUDA library ``libdckv_b200.so`` (sm_100a).  PyTorch supplies device memory and
streams.  If the library is missing the import of any entry point raises; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdckv_b200.so")
INCLUDE_DIR = os.path.join(os.path.dirname(_HERE), "include")

ROW_DIM = 6144
N_COEF = 2048
N_HIDDEN = 256
HEAD_KEPT = 4
TAIL_KEPT = 128

DCKV_OK, DCKV_EINVAL, DCKV_ECAPACITY, DCKV_ECUDA, DCKV_ECORRUPT, DCKV_ETIMEOUT, DCKV_ERANGE, DCKV_ESINGULAR = range(8)
STATUS_NAMES = {0: "OK", 1: "EINVAL", 2: "ECAPACITY", 3: "ECUDA", 4: "ECORRUPT", 5: "ETIMEOUT", 6: "ERANGE",
                7: "ESINGULAR"}

# fp64 layout of the closed-form fit's sums (include/dckv_fit.h)
FIT_OFF_GE = 0
FIT_OFF_CE = 2048 * 2048
FIT_OFF_GO = 2 * 2048 * 2048
FIT_OFF_CO = FIT_OFF_GO + 6144 * 6144
FIT_OFF_N = FIT_OFF_CO + 6144 * 2048
FIT_STATS_DOUBLES = FIT_OFF_N + 8

_lib = None


class DckvError(RuntimeError):
    def __init__(self, code, what):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)} ({code})")
        self.code = code


class _Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("mu", "basis", "w1", "w2", "delta", "laplace_b", "embed", "w_even", "w_odd")] + [
                   ("vocab", ctypes.c_int32), ("v1", ctypes.c_void_p), ("v2", ctypes.c_void_p)]


class ByteReport(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in
                ("total", "header_tables", "kept_rows", "states", "esc_counts", "esc_values", "words",
                 "padding", "payload")] + [(n, ctypes.c_uint32) for n in
                                           ("n_prompts", "n_chunks", "n_coded_rows", "n_escapes",
                                            "chunk_rows", "k_eff")]

    def as_dict(self):
        return {k: int(getattr(self, k)) for k, _ in self._fields_}


class WsView(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in ("q32", "qe", "cen8", "row_slot", "sym16", "q16", "x16", "g16", "counters")] + [
        ("n_rows", ctypes.c_int64), ("ne_pad", ctypes.c_int64), ("n_chunks", ctypes.c_int32),
        ("total", ctypes.c_uint64), ("code_width", ctypes.c_int32)]


def lib():
    """Load libdckv_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m learned_kv_cache_dckv_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "dckv_codec_create": (I, [ctypes.POINTER(_Params), I, I, ctypes.POINTER(P)]),
        "dckv_codec_destroy": (None, [P]),
        "dckv_codec_k_eff": (I, [P]),
        "dckv_workspace_bytes": (Z, [P, P, I]),
        "dckv_blob_bound": (Z, [P, P, I]),
        "dckv_encode": (I, [P, P, P, P, I, P, Z, P, P, P, Z, P]),
        "dckv_decode": (I, [P, P, Z, P, P, I, P, P, P, P, Z, P]),
        "dckv_decode_static": (I, [P, P, Z, P, P, I, P, P, P, P]),
        "dckv_bytes": (I, [P, Z, ctypes.POINTER(ByteReport)]),
        "dckv_last_error": (ctypes.c_char_p, []),
        "dckv_ws_offsets": (I, [P, P, I, I, ctypes.POINTER(WsView)]),
        "dckv_codec_export": (I, [P, P, P, P, P]),
        "dckv_codec_tables": (I, [P, ctypes.POINTER(P), ctypes.POINTER(P)]),
        "dckv_set_timing": (I, [P, I]),
        "dckv_get_timing": (I, [P, P, P, I]),
        "dckv_debug_gemm": (I, [I, P, I, P, I, I, I, P, I, I, P]),
        "dckv_debug_ratio": (I, [P, P]),
        "dckv_codec_info": (I, [P, P, P]),
        "dckv_codec_gemm_shape": (I, [P, P]),
        "dckv_launch_count": (ctypes.c_longlong, []),
        "dckv_fit_workspace_bytes": (Z, [P, P, I]),
        "dckv_fit_accumulate": (I, [P, P, ctypes.c_int32, P, P, P, I, P, P, P, Z, P]),
        "dckv_fit_solve_workspace_bytes": (Z, []),
        "dckv_fit_solve": (I, [P, ctypes.c_double, P, P, P, P, Z, P]),
        "dckv_fit_to_bf16": (I, [P, ctypes.c_int64, P, P]),
        "dckv_fit_scales_accumulate": (I, [P, P, P, P, I, P, P, P, Z, P]),
        "dckv_fit_scales_finish": (I, [P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def header_functions():
    """Names of every function declared in include/*.h."""
    names = []
    for fn in sorted(os.listdir(INCLUDE_DIR)):
        if fn.endswith(".h"):
            txt = open(os.path.join(INCLUDE_DIR, fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(dckv_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


def last_error() -> str:
    return lib().dckv_last_error().decode()


def _check(code, what):
    if code != DCKV_OK:
        raise DckvError(code, f"{what} ({last_error()})")


def _offs(seq_offsets):
    a = np.ascontiguousarray(np.asarray(seq_offsets, dtype=np.int64))
    return a, a.ctypes.data_as(ctypes.c_void_p), a.size - 1


def _ptr(t):
    """Device address of a tensor, or NULL for None (token ids of a codec without mean models)."""
    return None if t is None else t.data_ptr()


def _stream_ptr(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ---------------------------------------------------------------------------------- C ABI
def dckv_codec_create(params: dict, device: int = 0, chunk_rows: int = 0):
    """params: device tensors mu, basis, w1, w2, delta, laplace_b (fp32), embed, w_even,
    w_odd (bf16 or int16 holding bf16 bits), v1, v2 (fp32, optional); w1 / w2 None for a
    linear codec, embed / w_even / w_odd None for unconditional tables, v1 / v2 None for a
    linear synthesis.  Returns an opaque handle."""
    p = _Params()
    for k in ("mu", "basis", "w1", "w2", "delta", "laplace_b", "embed", "w_even", "w_odd", "v1", "v2"):
        v = params.get(k)
        setattr(p, k, None if v is None else v.data_ptr())
    p.vocab = 0 if params.get("embed") is None else int(params["embed"].shape[0])
    h = ctypes.c_void_p()
    _check(lib().dckv_codec_create(ctypes.byref(p), int(device), int(chunk_rows), ctypes.byref(h)),
           "dckv_codec_create")
    return h


def dckv_codec_destroy(handle):
    lib().dckv_codec_destroy(handle)


def dckv_codec_k_eff(handle) -> int:
    return int(lib().dckv_codec_k_eff(handle))


def dckv_workspace_bytes(handle, seq_offsets) -> int:
    a, ptr, b = _offs(seq_offsets)
    return int(lib().dckv_workspace_bytes(handle, ptr, b))


def dckv_blob_bound(handle, seq_offsets) -> int:
    a, ptr, b = _offs(seq_offsets)
    return int(lib().dckv_blob_bound(handle, ptr, b))


def dckv_encode(handle, rows, token_ids, seq_offsets, blob, blob_size, status, workspace, stream=None):
    """rows bf16 [sum N, 6144], token_ids int32 [sum N], blob uint8 (device), blob_size
    uint64[1]/int64[1] (device), status int32[1] (device), workspace uint8 (device)."""
    a, ptr, b = _offs(seq_offsets)
    _check(lib().dckv_encode(handle, rows.data_ptr(), _ptr(token_ids), ptr, b, blob.data_ptr(),
                             blob.numel() * blob.element_size(), blob_size.data_ptr(), status.data_ptr(),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream_ptr(stream)), "dckv_encode")


def dckv_decode(handle, blob, blob_bytes, token_ids, seq_offsets, k_out, v_out, status, workspace, stream=None):
    a, ptr, b = _offs(seq_offsets)
    _check(lib().dckv_decode(handle, blob.data_ptr(), int(blob_bytes), _ptr(token_ids), ptr, b,
                             k_out.data_ptr(), v_out.data_ptr(), status.data_ptr(), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), _stream_ptr(stream)), "dckv_decode")


def dckv_decode_static(handle, blob, blob_bytes, token_ids, seq_offsets, k_out, v_out, status, stream=None):
    """dckv_decode on the library's static per-device scratch (no workspace argument)."""
    a, ptr, b = _offs(seq_offsets)
    _check(lib().dckv_decode_static(handle, blob.data_ptr(), int(blob_bytes), _ptr(token_ids), ptr, b,
                                    k_out.data_ptr(), v_out.data_ptr(), status.data_ptr(), _stream_ptr(stream)),
           "dckv_decode_static")


def dckv_launch_count() -> int:
    return int(lib().dckv_launch_count())


def dckv_bytes(blob_host: bytes) -> dict:
    buf = ctypes.create_string_buffer(bytes(blob_host), len(blob_host))
    rep = ByteReport()
    _check(lib().dckv_bytes(buf, len(blob_host), ctypes.byref(rep)), "dckv_bytes")
    return rep.as_dict()


def dckv_ws_offsets(handle, seq_offsets, which: int) -> dict:
    a, ptr, b = _offs(seq_offsets)
    v = WsView()
    _check(lib().dckv_ws_offsets(handle, ptr, b, int(which), ctypes.byref(v)), "dckv_ws_offsets")
    return {k: int(getattr(v, k)) for k, _ in WsView._fields_}


def dckv_codec_export(handle):
    cdf = np.zeros((64, 510), np.uint16)
    scale = np.zeros(2048, np.uint8)
    keep = np.zeros(2048, np.uint8)
    exps = np.zeros(3, np.int32)
    _check(lib().dckv_codec_export(handle, cdf.ctypes.data_as(ctypes.c_void_p), scale.ctypes.data_as(ctypes.c_void_p),
                                   keep.ctypes.data_as(ctypes.c_void_p), exps.ctypes.data_as(ctypes.c_void_p)),
           "dckv_codec_export")
    return cdf, scale, keep, exps


def dckv_codec_tables(handle):
    te, to = ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib().dckv_codec_tables(handle, ctypes.byref(te), ctypes.byref(to)), "dckv_codec_tables")
    return te.value, to.value


def dckv_debug_ratio(handle, ratio_dev):
    _check(lib().dckv_debug_ratio(handle, None if ratio_dev is None else ratio_dev.data_ptr()), "dckv_debug_ratio")


def dckv_codec_info(handle):
    g = ctypes.c_int32()
    bits = ctypes.c_double()
    _check(lib().dckv_codec_info(handle, ctypes.byref(g), ctypes.byref(bits)), "dckv_codec_info")
    return {"chunk_rows": int(g.value), "model_bits_per_row": float(bits.value)}


def dckv_codec_gemm_shape(handle):
    a = (ctypes.c_int32 * 4)()
    _check(lib().dckv_codec_gemm_shape(handle, a), "dckv_codec_gemm_shape")
    return {"k_eff": a[0], "kw": a[1], "mp": a[2], "inv_lo_k": a[3]}


def dckv_set_timing(handle, enable: bool):
    _check(lib().dckv_set_timing(handle, 1 if enable else 0), "dckv_set_timing")


def dckv_get_timing(handle, max_stages: int = 24):
    ms = (ctypes.c_float * max_stages)()
    names = (ctypes.c_char_p * max_stages)()
    n = lib().dckv_get_timing(handle, ms, names, max_stages)
    return [(names[i].decode(), float(ms[i])) for i in range(max(0, n))]


def dckv_debug_gemm(bf16: bool, A, slabs: int, B, M: int, N: int, K: int, D, bn: int = 256, pair: bool = False,
                    stream=None):
    _check(lib().dckv_debug_gemm(1 if bf16 else 0, A.data_ptr(), int(slabs), B.data_ptr(), int(M), int(N), int(K),
                                 D.data_ptr(), int(bn), 1 if pair else 0, _stream_ptr(stream)), "dckv_debug_gemm")


# ---------------------------------------------------------------------------------- helpers
# ------------------------------------------------------------- closed-form fit (dckv_fit.h)
def dckv_fit_workspace_bytes(handle, seq_offsets) -> int:
    a, ptr, b = _offs(seq_offsets)
    return int(lib().dckv_fit_workspace_bytes(handle, ptr, b))


def dckv_fit_accumulate(handle, embed, rows, token_ids, seq_offsets, stats, status, workspace, stream=None):
    """embed bf16 [vocab, 2048] (device), rows bf16 [sum N, 6144], token_ids int32, stats fp64
    [FIT_STATS_DOUBLES] (accumulated into), status int32[1], workspace uint8 (device)."""
    a, ptr, b = _offs(seq_offsets)
    _check(lib().dckv_fit_accumulate(handle, embed.data_ptr(), int(embed.shape[0]), rows.data_ptr(),
                                     token_ids.data_ptr(), ptr, b, stats.data_ptr(), status.data_ptr(),
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                     _stream_ptr(stream)), "dckv_fit_accumulate")


def dckv_fit_solve_workspace_bytes() -> int:
    return int(lib().dckv_fit_solve_workspace_bytes())


def dckv_fit_solve(stats, ridge, w_even, w_odd, status, workspace, stream=None):
    """w_even fp64 [2048, 2048] and w_odd fp64 [6144, 2048] (device) receive the weights."""
    _check(lib().dckv_fit_solve(stats.data_ptr(), float(ridge), w_even.data_ptr(), w_odd.data_ptr(),
                                status.data_ptr(), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _stream_ptr(stream)),
           "dckv_fit_solve")


def dckv_fit_to_bf16(w, out, stream=None):
    """bf16 bits (out: int16/uint16-sized device tensor) of fp64 w, one RNE step."""
    _check(lib().dckv_fit_to_bf16(w.data_ptr(), int(w.numel()), out.data_ptr(), _stream_ptr(stream)),
           "dckv_fit_to_bf16")


def dckv_fit_scales_accumulate(handle, rows, token_ids, seq_offsets, abs_sum, status, workspace, stream=None):
    """abs_sum int64 [2049] (device), accumulated into."""
    a, ptr, b = _offs(seq_offsets)
    _check(lib().dckv_fit_scales_accumulate(handle, rows.data_ptr(), _ptr(token_ids), ptr, b, abs_sum.data_ptr(),
                                            status.data_ptr(), workspace.data_ptr(),
                                            workspace.numel() * workspace.element_size(), _stream_ptr(stream)),
           "dckv_fit_scales_accumulate")


def dckv_fit_scales_finish(handle, abs_sum, laplace_b, stream=None):
    _check(lib().dckv_fit_scales_finish(handle, abs_sum.data_ptr(), laplace_b.data_ptr(), _stream_ptr(stream)),
           "dckv_fit_scales_finish")


def upload_params(codec, device="cuda"):
    """Device tensors for dckv_codec_create from an object with numpy attributes mu, basis,
    w1, w2, delta, laplace_b (float32), embed, w_even, w_odd (bf16 bits as uint16) and,
    optionally, v1, v2 (float32)."""
    import torch

    out = {}
    for k in ("mu", "basis", "w1", "w2", "delta", "laplace_b", "v1", "v2"):
        v = getattr(codec, k, None)
        out[k] = None if v is None else torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(device)
    for k in ("embed", "w_even", "w_odd"):
        v = getattr(codec, k)
        if v is None:
            out[k] = None
            continue
        a = np.ascontiguousarray(v, np.uint16).view(np.int16)
        out[k] = torch.from_numpy(a).to(device).view(torch.bfloat16)
    return out


class Codec:
    """Owns a codec handle plus reusable workspace / blob / output buffers (torch)."""

    def __init__(self, params: dict, device: int = 0, chunk_rows: int = 0):
        import torch

        self.torch = torch
        self.device = torch.device("cuda", device)
        self.handle = dckv_codec_create(params, device, chunk_rows)
        self.params = params  # the library copies what it needs; kept alive for clarity
        self._ws = None
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.blob_size = torch.zeros(1, dtype=torch.int64, device=self.device)

    @property
    def k_eff(self):
        return dckv_codec_k_eff(self.handle)

    def workspace(self, seq_offsets):
        n = dckv_workspace_bytes(self.handle, seq_offsets)
        if n == 0:
            raise DckvError(DCKV_EINVAL, "dckv_workspace_bytes")
        if self._ws is None or self._ws.numel() < n:
            self._ws = self.torch.empty(n, dtype=self.torch.uint8, device=self.device)
        return self._ws

    def encode(self, rows, token_ids, seq_offsets, blob=None, stream=None):
        if blob is None:
            blob = self.torch.empty(dckv_blob_bound(self.handle, seq_offsets), dtype=self.torch.uint8,
                                    device=self.device)
        ws = self.workspace(seq_offsets)
        dckv_encode(self.handle, rows, token_ids, seq_offsets, blob, self.blob_size, self.status, ws, stream)
        return blob

    def decode(self, blob, blob_bytes, token_ids, seq_offsets, k_out=None, v_out=None, stream=None):
        n_tok = int(np.asarray(seq_offsets)[-1])
        if k_out is None:
            k_out = self.torch.empty((6, n_tok, 2, 256), dtype=self.torch.bfloat16, device=self.device)
        if v_out is None:
            v_out = self.torch.empty((6, n_tok, 2, 256), dtype=self.torch.bfloat16, device=self.device)
        ws = self.workspace(seq_offsets)
        dckv_decode(self.handle, blob, blob_bytes, token_ids, seq_offsets, k_out, v_out, self.status, ws, stream)
        return k_out, v_out

    def workspace_codes(self, seq_offsets, which: int = 0, rows=None):
        """Codes the last encode (which=0: q32, int32) or decode (which=1: q16, fp16 as float32)
        left in the workspace, as numpy [rows][2048] by component (the library keeps kept
        components only, compact; dropped components are 0).  rows: coded-row indices (all
        if None)."""
        torch = self.torch
        v = dckv_ws_offsets(self.handle, seq_offsets, which)
        n, k = v["n_rows"], self.k_eff
        if which == 0:
            c = self._ws[v["q32"]: v["q32"] + 4 * n * 2048].view(torch.int32).reshape(n, 2048)
        else:
            c = self._ws[v["q16"]: v["q16"] + 2 * n * 2048].view(torch.float16).reshape(n, 2048).float()
        if rows is not None:
            c = c[torch.as_tensor(np.asarray(rows, np.int64), device=c.device)]
        c = c[:, :k].cpu().numpy()
        keep = dckv_codec_export(self.handle)[2].astype(bool)
        out = np.zeros((c.shape[0], 2048), c.dtype)
        out[:, keep] = c
        return out

    def close(self):
        if self.handle is not None:
            dckv_codec_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
