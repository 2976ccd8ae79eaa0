"""Thin ctypes binding of liborbitquant.so (argument marshalling only).

Every step of the hot path runs in the library's CUDA kernels; this module
only turns torch tensors into device pointers and sizes, picks the current
torch stream, and turns non-zero status codes into exceptions.  There is no
fallback: if the shared library is missing, importing this module fails.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liborbitquant.so")

OQ_OK, OQ_ERR_ARG, OQ_ERR_UNSUPPORTED, OQ_ERR_ALIGN, OQ_ERR_CUDA, OQ_ERR_TIMEOUT, OQ_ERR_NOMEM = range(7)
EPILOGUES = {"none": 0, "gelu": 1}
ROTATIONS = {"rpbh": 0, "block_rht": 1, "full_rht": 2}  # OQ_ROT_*

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m calibration_free_rotated_b200.build` "
        "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

_c_int, _c_void_p, _c_size_t = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
_SIGS = {
    "oq_version": (_c_int, []),
    "oq_device_allocations": (ctypes.c_longlong, []),
    "oq_last_error": (ctypes.c_char_p, []),
    "oq_get_device_status": (_c_int, [_c_void_p]),
    "oq_make_rpbh": (_c_int, [ctypes.c_uint64, _c_int, _c_int, ctypes.POINTER(_c_void_p)]),
    "oq_make_rotation": (_c_int, [ctypes.c_uint64, _c_int, _c_int, _c_int, ctypes.POINTER(_c_void_p)]),
    "oq_rotation_kind": (_c_int, [_c_void_p, ctypes.POINTER(_c_int)]),
    "oq_make_composed_rpbh": (_c_int, [ctypes.c_uint64, _c_int, _c_int, _c_int, ctypes.POINTER(_c_void_p)]),
    "oq_rotation_rounds": (_c_int, [_c_void_p, ctypes.POINTER(_c_int)]),
    "oq_rpbh_export_round": (_c_int, [_c_void_p, _c_int, _c_void_p, _c_void_p]),
    "oq_rpbh_info": (_c_int, [_c_void_p, ctypes.POINTER(_c_int), ctypes.POINTER(_c_int)]),
    "oq_rpbh_export": (_c_int, [_c_void_p, _c_void_p, _c_void_p]),
    "oq_free_rpbh": (None, [_c_void_p]),
    "oq_build_codebook": (_c_int, [_c_int, _c_int, ctypes.POINTER(_c_void_p)]),
    "oq_codebook_info": (_c_int, [_c_void_p, ctypes.POINTER(_c_int), ctypes.POINTER(_c_int)]),
    "oq_codebook_export": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, ctypes.POINTER(_c_int),
                                    ctypes.POINTER(ctypes.c_double)]),
    "oq_free_codebook": (None, [_c_void_p]),
    "oq_quantize_act": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p]),
    "oq_quantize_weight": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p]),
    "oq_linear_codes": (_c_int, [_c_int, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p,
                                 _c_int, _c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p]),
    "oq_linear_workspace_bytes": (_c_size_t, [_c_int, _c_int, _c_int]),
    "oq_row_flatness": (_c_int, [_c_void_p, _c_int, _c_int, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "oq_linear": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p, _c_int,
                           _c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_void_p]),
    "oq_linear_noalloc": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p,
                                   _c_int, _c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p]),
    "oq_test_composed_tables": (_c_int, [_c_void_p, _c_int, _c_void_p, _c_void_p, _c_void_p]),
}
NOALLOC_SCRATCH_BYTES = 32 << 20
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class OQError(RuntimeError):
    def __init__(self, code, message):
        super().__init__(f"orbitquant error {code}: {message}")
        self.code = code


def _check(rc):
    if rc != OQ_OK:
        raise OQError(rc, _lib.oq_last_error().decode())


def lib():
    """The loaded ctypes library (for tests that call the C ABI directly)."""
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Rpbh:
    """Handle of the RPBH rotation for one (seed, d, block); `kind` selects a
    variant of the rotation ablation ("rpbh", "block_rht", "full_rht");
    `rounds` > 1 composes that many RPBH rounds (oq_make_composed_rpbh)."""

    def __init__(self, seed: int, d: int, block: int = 0, kind: str = "rpbh", rounds: int = 1):
        h = ctypes.c_void_p()
        if rounds == 1:
            _check(_lib.oq_make_rotation(seed, d, block, ROTATIONS[kind], ctypes.byref(h)))
        else:
            if kind != "rpbh":
                raise ValueError("composed rounds are RPBH rounds")
            _check(_lib.oq_make_composed_rpbh(seed, d, block, rounds, ctypes.byref(h)))
        self._h = h
        dd, bb, kk, rr = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        _check(_lib.oq_rpbh_info(h, ctypes.byref(dd), ctypes.byref(bb)))
        _check(_lib.oq_rotation_kind(h, ctypes.byref(kk)))
        _check(_lib.oq_rotation_rounds(h, ctypes.byref(rr)))
        self.seed, self.d, self.block, self.rounds = seed, dd.value, bb.value, rr.value
        self.kind = {v: k for k, v in ROTATIONS.items()}[kk.value]

    @property
    def handle(self):
        return self._h

    def export(self):
        import numpy as np
        perm = np.empty(self.d, dtype=np.int32)
        signs = np.empty((self.d + 31) // 32, dtype=np.uint32)
        _check(_lib.oq_rpbh_export(self._h, perm.ctypes.data, signs.ctypes.data))
        return perm, signs

    def export_round(self, rnd: int):
        """(perm, sign words) of round `rnd` (1-based) of a composed rotation."""
        import numpy as np
        perm = np.empty(self.d, dtype=np.int32)
        signs = np.empty((self.d + 31) // 32, dtype=np.uint32)
        _check(_lib.oq_rpbh_export_round(self._h, rnd, perm.ctypes.data, signs.ctypes.data))
        return perm, signs

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and _lib is not None:
            _lib.oq_free_rpbh(h)


class Codebook:
    """Handle of the Lloyd-Max codebook C^(d,b)."""

    def __init__(self, d: int, bits: int):
        h = ctypes.c_void_p()
        _check(_lib.oq_build_codebook(d, bits, ctypes.byref(h)))
        self._h = h
        self.d, self.bits = d, bits

    @property
    def handle(self):
        return self._h

    def export(self):
        import numpy as np
        L = 1 << self.bits
        c = np.empty(L, dtype=np.float64)
        b = np.empty(L - 1, dtype=np.float64)
        lut = np.empty(L, dtype=np.uint16)
        it = ctypes.c_int()
        dist = ctypes.c_double()
        _check(_lib.oq_codebook_export(self._h, c.ctypes.data, b.ctypes.data, lut.ctypes.data,
                                       ctypes.byref(it), ctypes.byref(dist)))
        return {"centroids": c, "boundaries": b, "lut_fp16": lut, "iterations": it.value,
                "distortion": dist.value}

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and _lib is not None:
            _lib.oq_free_codebook(h)


def code_bytes(d: int, bits: int) -> int:
    return d * bits // 8


def quantize_act(rpbh: Rpbh, cb: Codebook, X: torch.Tensor, codes=None, norms=None, stream=None):
    """X: cuda bf16 [M, d] -> (codes uint8 [M, d*b/8], norms float32 [M])."""
    M = X.shape[0]
    if codes is None:
        codes = torch.empty((M, code_bytes(rpbh.d, cb.bits)), dtype=torch.uint8, device=X.device)
    if norms is None:
        norms = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check(_lib.oq_quantize_act(rpbh.handle, cb.handle, _ptr(X), M, _ptr(codes), _ptr(norms), _stream(stream)))
    return codes, norms


def quantize_weight(rpbh: Rpbh, cb: Codebook, W: torch.Tensor, codes=None, norms=None, stream=None):
    """W: cuda bf16 [N, d] -> (codes uint8 [N, d*b/8], norms bf16 [N])."""
    N = W.shape[0]
    if codes is None:
        codes = torch.empty((N, code_bytes(rpbh.d, cb.bits)), dtype=torch.uint8, device=W.device)
    if norms is None:
        norms = torch.empty((N,), dtype=torch.bfloat16, device=W.device)
    _check(_lib.oq_quantize_weight(rpbh.handle, cb.handle, _ptr(W), N, _ptr(codes), _ptr(norms), _stream(stream)))
    return codes, norms


def linear_codes(d, cb_a: Codebook, cb_w: Codebook, a_codes, a_norm, w_codes, w_norm, bias=None, epilogue="none",
                 out_f32=None, out_bf16=None, want_f32=True, want_bf16=False, stream=None):
    M, N = a_codes.shape[0], w_codes.shape[0]
    dev = a_codes.device
    if out_f32 is None and want_f32:
        out_f32 = torch.empty((M, N), dtype=torch.float32, device=dev)
    if out_bf16 is None and want_bf16:
        out_bf16 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _check(_lib.oq_linear_codes(d, cb_a.handle, cb_w.handle, _ptr(a_codes), _ptr(a_norm), M, _ptr(w_codes),
                                _ptr(w_norm), N, _ptr(bias), EPILOGUES[epilogue], _ptr(out_f32), _ptr(out_bf16),
                                _stream(stream)))
    return out_f32, out_bf16


def row_flatness(X, rho3=None, rhoinf=None, batch_max=None, want_rows=True, stream=None):
    """Flatness check of the rows of X (cuda bf16 [M, d]): per-row rho3 and
    rhoinf (float [M] each, unless want_rows is False) and their batch maxima
    (float [2])."""
    M, d = X.shape
    dev = X.device
    if want_rows:
        rho3 = torch.empty((M,), dtype=torch.float32, device=dev) if rho3 is None else rho3
        rhoinf = torch.empty((M,), dtype=torch.float32, device=dev) if rhoinf is None else rhoinf
    batch_max = torch.empty((2,), dtype=torch.float32, device=dev) if batch_max is None else batch_max
    _check(_lib.oq_row_flatness(_ptr(X), M, d, _ptr(rho3), _ptr(rhoinf), _ptr(batch_max), _stream(stream)))
    return rho3, rhoinf, batch_max


def workspace_bytes(M: int, d: int, bits_a: int) -> int:
    return int(_lib.oq_linear_workspace_bytes(M, d, bits_a))


def linear(rpbh: Rpbh, cb_a: Codebook, cb_w: Codebook, X, w_codes, w_norm, bias=None, epilogue="none",
           out_f32=None, out_bf16=None, want_f32=True, want_bf16=False, workspace=None, stream=None):
    """Full layer: act-quant of X (cuda bf16 [M, d]) then the codebook GEMM."""
    M, N = X.shape[0], w_codes.shape[0]
    dev = X.device
    if out_f32 is None and want_f32:
        out_f32 = torch.empty((M, N), dtype=torch.float32, device=dev)
    if out_bf16 is None and want_bf16:
        out_bf16 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    need = workspace_bytes(M, rpbh.d, cb_a.bits)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=dev)
    _check(_lib.oq_linear(rpbh.handle, cb_a.handle, cb_w.handle, _ptr(X), M, _ptr(w_codes), _ptr(w_norm), N,
                          _ptr(bias), EPILOGUES[epilogue], _ptr(out_f32), _ptr(out_bf16), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream)))
    return out_f32, out_bf16


def device_status(stream=None):
    """Raises OQError if a kernel's bounded wait gave up since the last call."""
    _check(_lib.oq_get_device_status(_stream(stream)))


def device_allocations() -> int:
    """How many device allocations the library has made in this process."""
    return int(_lib.oq_device_allocations())


def linear_noalloc(rpbh: Rpbh, cb_a: Codebook, cb_w: Codebook, X, w_codes, w_norm, bias=None, epilogue="none",
                   out_f32=None, out_bf16=None, stream=None):
    """oq_linear_noalloc: the full layer with the library's static scratch
    instead of a workspace.  Outputs must be passed in (this call is for code
    that cannot allocate)."""
    M, N = X.shape[0], w_codes.shape[0]
    _check(_lib.oq_linear_noalloc(rpbh.handle, cb_a.handle, cb_w.handle, _ptr(X), M, _ptr(w_codes), _ptr(w_norm),
                                  N, _ptr(bias), EPILOGUES[epilogue], _ptr(out_f32), _ptr(out_bf16),
                                  _stream(stream)))
    return out_f32, out_bf16
