"""ctypes binding of ``libflashloop.so`` (declared in ``include/flashloop.h``).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch provides device memory (the workspace and the weight tensors)
and streams.  Loading fails loudly when the library is missing; there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflashloop.so")

FL_OK = 0
FL_OPT_USE_GRAPH = 1
FL_OPT_PROFILE = 2
FL_OPT_PDL = 3
FL_OPT_GEMM_TIMES = 5
FL_OPT_TC_PREFILL = 6
FL_OPT_CORR_CLUSTER = 7
KINDS = ["gemm", "attn", "dscore", "correct", "kv", "select", "norm", "other"]
STATUS = {0: "ok", 1: "invalid argument", 2: "capacity exceeded", 3: "workspace", 4: "cuda error",
          5: "timeout", 6: "nonfinite", 7: "unsupported"}


class FlashLoopError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status}) {detail}".strip())
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("n_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("ffn_dim", ctypes.c_int), ("n_layers", ctypes.c_int),
                ("n_loops", ctypes.c_int), ("rho", ctypes.c_double), ("c_cols", ctypes.c_int),
                ("q_tile", ctypes.c_int), ("resid_bits", ctypes.c_int), ("group_size", ctypes.c_int),
                ("resid_scale", ctypes.c_float), ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("vocab", ctypes.c_int), ("max_batch", ctypes.c_int), ("max_ctx", ctypes.c_int),
                ("max_tokens", ctypes.c_int), ("kv_mode", ctypes.c_int), ("n_prelude", ctypes.c_int),
                ("n_coda", ctypes.c_int), ("loop_embed", ctypes.c_int), ("inject_scale", ctypes.c_float),
                ("resid_rows", ctypes.c_int)]


LAYER_FIELDS = ("attn_norm", "w_qkv", "w_o", "mlp_norm", "w_gate", "w_up", "w_down")


class Layers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LAYER_FIELDS]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LAYER_FIELDS + ("final_norm", "w_out")] + [
        ("prelude", Layers), ("coda", Layers), ("loop_embed", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SIG = {
    "flashloop_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(Config)]),
    "flashloop_init": (_I, [ctypes.POINTER(Config), ctypes.POINTER(Weights), _P, ctypes.c_size_t, _P,
                            ctypes.POINTER(_P)]),
    "flashloop_prefill": (_I, [_P, _P, _I, _I, _P, _P, _P]),
    "flashloop_decode_step": (_I, [_P, _P, _I, _P, _P, _P]),
    "flashloop_kv_bytes": (_I, [_P, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_double),
                                ctypes.POINTER(ctypes.c_double)]),
    "flashloop_kv_bytes_for": (_I, [ctypes.POINTER(Config), ctypes.POINTER(ctypes.c_size_t),
                                    ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
    "flashloop_reset": (_I, [_P, _P, _P]),
    "flashloop_sync_status": (_I, [_P, _P]),
    "flashloop_destroy": (None, [_P]),
    "flashloop_status_string": (ctypes.c_char_p, [_I]),
    "flashloop_last_cuda_error": (ctypes.c_char_p, [_P]),
    "flashloop_import_lazy": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "flashloop_import_dense": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "flashloop_import_extra": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "flashloop_export_slice": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "flashloop_force_selection": (_I, [_P, _P, _I, _I, _P, _P, _I]),
    "flashloop_read_trace": (_I, [_P, _P, _P, _P, _P, _P]),
    "flashloop_set_trace": (_I, [_P, _P, _I, _P, _I]),
    "flashloop_force_codes": (_I, [_P, _P, _P, _I]),
    "flashloop_set_option": (_I, [_P, _I, _I]),
    "flashloop_profile": (_I, [_P, _P, _P, _P]),
    "flashloop_kernels_per_call": (_I, [_P]),
    "flashloop_gemm_times": (_I, [_P, _P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I)]),
    "fl_test_topk": (_I, [_P, _I, _I, _I, _P, _P]),
    "fl_test_quantize": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
    "fl_test_quantize_residual": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "fl_test_gemm_scratch_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "fl_test_gemm": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, ctypes.c_size_t, _P]),
    "fl_gemm_skinny_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FileNotFoundError(f"{LIB_PATH} is missing: run `python -m cross_loop_sparsity_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIG.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(st: int, what: str, ctx=None):
    if st != FL_OK:
        e = lib().flashloop_last_cuda_error(ctx)
        detail = e.decode() if e else ""
        raise FlashLoopError(st, what, detail)


def make_config(cfg, max_batch: int, max_ctx: int, max_tokens: int = 0, resid_bits: int | None = None) -> Config:
    """Fill the C config from a ``synth.LoopConfig``-like object."""
    return Config(cfg.d_model, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn_dim, cfg.n_layers, cfg.n_loops,
                  float(cfg.rho), cfg.c_cols, cfg.q_tile, cfg.resid_bits if resid_bits is None else resid_bits,
                  cfg.group_size, float(cfg.resid_scale), float(cfg.rms_eps), float(cfg.rope_theta), cfg.vocab,
                  max_batch, max_ctx, max_tokens, int(getattr(cfg, "kv_mode", 0)),
                  int(getattr(cfg, "n_prelude", 0)), int(getattr(cfg, "n_coda", 0)),
                  int(getattr(cfg, "loop_embed", 0)), float(getattr(cfg, "inject_scale", 0.0)),
                  int(getattr(cfg, "resid_rows", 0)))


def workspace_bytes(c: Config) -> int:
    return int(lib().flashloop_workspace_bytes(ctypes.byref(c)))


def kv_bytes_for(c: Config):
    tot, per, dense = ctypes.c_size_t(), ctypes.c_double(), ctypes.c_double()
    _check(lib().flashloop_kv_bytes_for(ctypes.byref(c), ctypes.byref(tot), ctypes.byref(per), ctypes.byref(dense)),
           "kv_bytes_for")
    return int(tot.value), per.value, dense.value


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    return None if stream is None else ctypes.c_void_p(stream.cuda_stream)


def upload_weights(w: dict, device="cuda"):
    """Stack the generator's per-layer weights into device tensors (bf16 bits as int16)."""
    import torch

    def stack(layers, name, dt=np.uint16):
        a = np.stack([lw[name] for lw in layers]).astype(dt, copy=False)
        if dt == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(device)
        return torch.from_numpy(a).to(device)

    def layer_stack(layers):
        return {n: stack(layers, n, np.float32 if n.endswith("norm") else np.uint16) for n in LAYER_FIELDS}

    out = layer_stack(w["layers"])
    out["final_norm"] = torch.from_numpy(np.asarray(w["final_norm"], np.float32)).to(device)
    out["w_out"] = torch.from_numpy(np.asarray(w["w_out"]).view(np.int16)).to(device)
    for part in ("prelude", "coda"):
        if w.get(part):
            out[part] = layer_stack(w[part])
    if "loop_embed" in w:
        out["loop_embed"] = torch.from_numpy(np.asarray(w["loop_embed"], np.float32)).to(device)
    return out


class FlashLoop:
    """One context: a KV cache and the per-call state in a torch-owned workspace."""

    def __init__(self, cfg, dev_weights: dict, max_batch: int, max_ctx: int, max_tokens: int = 0,
                 resid_bits: int | None = None, stream=None):
        import torch
        self.cfg = cfg
        self.c = make_config(cfg, max_batch, max_ctx, max_tokens, resid_bits)
        self.weights = dev_weights  # keep alive: the library borrows these pointers
        nbytes = workspace_bytes(self.c)
        if nbytes == 0:
            raise FlashLoopError(1, "workspace_bytes", "invalid config")
        self.workspace = torch.empty(nbytes + 256, dtype=torch.uint8, device="cuda")
        off = (-self.workspace.data_ptr()) % 256
        self._ws_ptr = self.workspace.data_ptr() + off
        self._ws_bytes = nbytes
        def layers(d):
            return Layers(*[d[n].data_ptr() for n in LAYER_FIELDS]) if d else Layers()

        wt = Weights(*[dev_weights[n].data_ptr() for n in LAYER_FIELDS + ("final_norm", "w_out")],
                     layers(dev_weights.get("prelude")), layers(dev_weights.get("coda")),
                     dev_weights["loop_embed"].data_ptr() if "loop_embed" in dev_weights else None)
        self._wstruct = wt
        ctx = ctypes.c_void_p()
        st = lib().flashloop_init(ctypes.byref(self.c), ctypes.byref(wt), ctypes.c_void_p(self._ws_ptr),
                                  ctypes.c_size_t(nbytes), _stream_ptr(stream), ctypes.byref(ctx))
        _check(st, "flashloop_init")
        self.ctx = ctx
        self.lazy = self.c.resid_bits != 16

    def close(self):
        if getattr(self, "ctx", None):
            lib().flashloop_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- calls ---------------------------------------------------------------
    def prefill(self, h0, B: int, T: int, h_out=None, logits=None, stream=None):
        _check(lib().flashloop_prefill(self.ctx, _ptr(h0), B, T, _ptr(h_out), _ptr(logits), _stream_ptr(stream)),
               "flashloop_prefill", self.ctx)

    def decode_step(self, h0, B: int, h_out=None, logits=None, stream=None):
        _check(lib().flashloop_decode_step(self.ctx, _ptr(h0), B, _ptr(h_out), _ptr(logits), _stream_ptr(stream)),
               "flashloop_decode_step", self.ctx)

    def kv_bytes(self):
        tot, per, dense = ctypes.c_size_t(), ctypes.c_double(), ctypes.c_double()
        _check(lib().flashloop_kv_bytes(self.ctx, ctypes.byref(tot), ctypes.byref(per), ctypes.byref(dense)),
               "flashloop_kv_bytes")
        return int(tot.value), per.value, dense.value

    def reset(self, lens=None, stream=None):
        arr = None
        if lens is not None:
            v = np.zeros(self.c.max_batch, np.int32)
            v[:len(lens)] = np.asarray(lens, np.int32)
            arr = v.ctypes.data_as(ctypes.c_void_p)
            self._lens_keep = v
        _check(lib().flashloop_reset(self.ctx, arr, _stream_ptr(stream)), "flashloop_reset", self.ctx)

    def sync_status(self, stream=None) -> int:
        return int(lib().flashloop_sync_status(self.ctx, _stream_ptr(stream)))

    def profile(self, stream=None):
        """{kind: (ms, launches)} of the last call made with FL_OPT_PROFILE on."""
        ms = (ctypes.c_float * len(KINDS))()
        n = (ctypes.c_int * len(KINDS))()
        _check(lib().flashloop_profile(self.ctx, _stream_ptr(stream), ms, n), "flashloop_profile", self.ctx)
        return {k: (float(ms[i]), int(n[i])) for i, k in enumerate(KINDS)}

    def gemm_times(self, stream=None):
        """(summed device ms, launches) of the last call's GEMMs (FL_OPT_GEMM_TIMES on)."""
        ms, n = ctypes.c_double(), ctypes.c_int()
        _check(lib().flashloop_gemm_times(self.ctx, _stream_ptr(stream), ctypes.byref(ms), ctypes.byref(n)),
               "gemm_times", self.ctx)
        return ms.value, n.value

    def kernels_per_call(self) -> int:
        return int(lib().flashloop_kernels_per_call(self.ctx))

    def set_option(self, opt: int, value: int):
        _check(lib().flashloop_set_option(self.ctx, opt, value), "flashloop_set_option")

    # -- cache import / export --------------------------------------------------
    def import_lazy(self, layer, seq, base_k, base_v, codes_k, codes_v, scales_k, scales_v, stream=None):
        n = base_k.shape[1]
        _check(lib().flashloop_import_lazy(self.ctx, layer, seq, n, _ptr(base_k), _ptr(base_v), _ptr(codes_k),
                                           _ptr(codes_v), _ptr(scales_k), _ptr(scales_v), _stream_ptr(stream)),
               "flashloop_import_lazy", self.ctx)

    def import_dense(self, layer, seq, kv_k, kv_v, stream=None):
        n = kv_k.shape[2]
        _check(lib().flashloop_import_dense(self.ctx, layer, seq, n, _ptr(kv_k), _ptr(kv_v), _stream_ptr(stream)),
               "flashloop_import_dense", self.ctx)

    def load_context(self, ctx: dict, dense: bool = False):
        """Import a cache given as host arrays (the layout ``synth.make_context`` /
        ``make_dense_context`` returns) slice by slice, then set the lengths."""
        import torch
        cfg = self.cfg
        lens = ctx["lens"]
        for j in range(cfg.n_layers):
            for b, n in enumerate(lens):
                n = int(n)
                if n == 0:
                    continue
                if dense:
                    kk = torch.from_numpy(np.ascontiguousarray(ctx["kv_k"][j, :, b, :, :n]).view(np.int16)).cuda()
                    vv = torch.from_numpy(np.ascontiguousarray(ctx["kv_v"][j, :, b, :, :n]).view(np.int16)).cuda()
                    self.import_dense(j, b, kk, vv)
                    continue
                a = {}
                for nm in ("k", "v"):
                    a["base_" + nm] = torch.from_numpy(
                        np.ascontiguousarray(ctx["base_" + nm][j, b, :, :n]).view(np.int16)).cuda()
                    a["codes_" + nm] = torch.from_numpy(np.ascontiguousarray(ctx["codes_" + nm][j, :, b, :, :n])).cuda()
                    a["scales_" + nm] = torch.from_numpy(
                        np.ascontiguousarray(ctx["scales_" + nm][j, :, b, :, :n]).view(np.int16)).cuda()
                self.import_lazy(j, b, a["base_k"], a["base_v"], a["codes_k"], a["codes_v"], a["scales_k"],
                                 a["scales_v"])
                torch.cuda.synchronize()   # the import copies read the staged tensors
        if "extra_k" in ctx:             # the prelude / coda layers' one-pass KV
            for x in range(ctx["extra_k"].shape[0]):
                for b, n in enumerate(lens):
                    n = int(n)
                    if n == 0:
                        continue
                    kk = torch.from_numpy(np.ascontiguousarray(ctx["extra_k"][x, b, :, :n]).view(np.int16)).cuda()
                    vv = torch.from_numpy(np.ascontiguousarray(ctx["extra_v"][x, b, :, :n]).view(np.int16)).cuda()
                    _check(lib().flashloop_import_extra(self.ctx, x, b, n, _ptr(kk), _ptr(vv), None),
                           "flashloop_import_extra", self.ctx)
                    torch.cuda.synchronize()
        torch.cuda.synchronize()
        self.reset([int(x) for x in lens])
        torch.cuda.synchronize()

    def load_context_device(self, lens, seed=None, dense: bool = False):
        """Import a synthetic context drawn on the device (``synth.context_slices_device``)
        slice by slice, then set the lengths."""
        import torch
        from cross_loop_sparsity_b200 import synth
        for sl in synth.context_slices_device(self.cfg, lens, seed=seed, dense=dense):
            if dense:
                self.import_dense(*sl)
            else:
                self.import_lazy(*sl)
            torch.cuda.synchronize()    # the import copies read the drawn tensors
        self.reset([int(x) for x in lens])
        torch.cuda.synchronize()

    def export_slice(self, layer, loop, seq, which, n, stream=None):
        """Returns (codes, scales) numpy arrays; loop 1 (or dense) returns (bf16 bits [Hkv][n][hd], None)."""
        import torch
        c = self.c
        if not self.lazy or loop == 1:
            out = torch.empty((c.n_kv_heads, n, c.head_dim), dtype=torch.int16, device="cuda")
            _check(lib().flashloop_export_slice(self.ctx, layer, loop, seq, which, n, _ptr(out), None,
                                                _stream_ptr(stream)), "export", self.ctx)
            torch.cuda.synchronize()
            return out.cpu().numpy().view(np.uint16), None
        rb = c.head_dim * c.resid_bits // 8
        codes = torch.empty((c.n_kv_heads, n, rb), dtype=torch.uint8, device="cuda")
        scales = torch.empty((c.n_kv_heads, n, c.head_dim // c.group_size), dtype=torch.int16, device="cuda")
        _check(lib().flashloop_export_slice(self.ctx, layer, loop, seq, which, n, _ptr(codes), _ptr(scales),
                                            _stream_ptr(stream)), "export", self.ctx)
        torch.cuda.synchronize()
        return codes.cpu().numpy(), scales.cpu().numpy().view(np.float16)

    def force_selection(self, sel=None, cols=None, ncols=None, n_tiles: int = 0):
        """sel int32 [K-1][n_sel] and/or cols int32 [M][n_tiles][Hkv][c] with
        ncols [M][n_tiles][Hkv]; a part left None stays free; all None clears."""
        sel_p, n_loops, n_sel = None, 0, 0
        cols_p = ncols_p = None
        keep = []
        if sel is not None:
            sel = np.ascontiguousarray(sel, np.int32)
            keep.append(sel)
            sel_p, n_loops, n_sel = sel.ctypes.data_as(ctypes.c_void_p), sel.shape[0], sel.shape[1]
        if cols is not None:
            cols = np.ascontiguousarray(cols, np.int32)
            ncols = np.ascontiguousarray(ncols, np.int32)
            keep += [cols, ncols]
            cols_p, ncols_p = cols.ctypes.data_as(ctypes.c_void_p), ncols.ctypes.data_as(ctypes.c_void_p)
        self._forced_keep = keep
        _check(lib().flashloop_force_selection(self.ctx, sel_p, n_loops, n_sel, cols_p, ncols_p,
                                               n_tiles if cols is not None else 0),
               "force_selection", self.ctx)

    def force_codes(self, codes=None, scales=None):
        """codes int8 [M][K-1][n_sel][2][Hkv][hd], scales float16 [M][K-1][n_sel][2][Hkv][hd/g]; None clears."""
        if codes is None:
            _check(lib().flashloop_force_codes(self.ctx, None, None, 0), "force_codes")
            return
        codes = np.ascontiguousarray(codes, np.int8)
        scales = np.ascontiguousarray(scales, np.float16).view(np.uint16)
        self._forced_codes_keep = (codes, scales)
        _check(lib().flashloop_force_codes(self.ctx, codes.ctypes.data_as(ctypes.c_void_p),
                                           scales.ctypes.data_as(ctypes.c_void_p), codes.shape[2]),
               "force_codes", self.ctx)

    def set_trace(self, kv_rows=None, n_slots: int = 0, col_keys=None, n_tiles: int = 0):
        """Check buffers (cuda float32 tensors, or None): kv_rows [M][K-1][n_slots][2][Hkv][hd]
        receives the new K/V rows each lazy loop quantised; col_keys [M][n_tiles][Hkv][max_ctx]
        the delta-score keys of every column set the call chose."""
        self._trace_keep = (kv_rows, col_keys)
        _check(lib().flashloop_set_trace(self.ctx, None if kv_rows is None else _ptr(kv_rows), n_slots,
                                         None if col_keys is None else _ptr(col_keys), n_tiles),
               "set_trace", self.ctx)

    def read_trace(self, N: int, n_sel: int, n_tiles: int, stream=None):
        c = self.c
        L = c.n_loops - 1
        sel = np.zeros((L, n_sel), np.int32)
        keys = np.zeros((L, N), np.float32)
        cols = np.zeros((c.n_layers, n_tiles, c.n_kv_heads, c.c_cols), np.int32)
        ncols = np.zeros((c.n_layers, n_tiles, c.n_kv_heads), np.int32)
        _check(lib().flashloop_read_trace(self.ctx, sel.ctypes.data_as(ctypes.c_void_p),
                                          keys.ctypes.data_as(ctypes.c_void_p), cols.ctypes.data_as(ctypes.c_void_p),
                                          ncols.ctypes.data_as(ctypes.c_void_p), _stream_ptr(stream)),
               "read_trace", self.ctx)
        return sel, keys, cols, ncols


# ---------------------------------------------------------------------------- unit entry points
def topk(keys, k: int, stream=None):
    """keys: cuda float32 [n_seg, n]; returns cuda int32 [n_seg, min(k, n)]."""
    import torch
    n_seg, n = keys.shape
    out = torch.empty((n_seg, min(k, n)), dtype=torch.int32, device=keys.device)
    _check(lib().fl_test_topk(_ptr(keys), n_seg, n, k, _ptr(out), _stream_ptr(stream)), "fl_test_topk")
    return out


def quantize(r, g: int, bits: int, stream=None):
    """r: cuda float32 [rows, width]; returns (packed codes uint8, fp16 scale bits int16)."""
    import torch
    rows, width = r.shape
    codes = torch.empty((rows, width * bits // 8), dtype=torch.uint8, device=r.device)
    scales = torch.empty((rows, width // g), dtype=torch.int16, device=r.device)
    _check(lib().fl_test_quantize(_ptr(r), rows, width, g, bits, _ptr(codes), _ptr(scales), _stream_ptr(stream)),
           "fl_test_quantize")
    return codes, scales


def quantize_residual(x, prev, g: int, bits: int, stream=None):
    """x: cuda float32 [rows, width], prev: cuda bf16 (or int16 bits) [rows, width]; quantises
    r = x - prev; returns (packed codes uint8, fp16 scale bits int16)."""
    import torch
    rows, width = x.shape
    codes = torch.empty((rows, width * bits // 8), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, width // g), dtype=torch.int16, device=x.device)
    _check(lib().fl_test_quantize_residual(_ptr(x), _ptr(prev), rows, width, g, bits, _ptr(codes), _ptr(scales),
                                           _stream_ptr(stream)), "fl_test_quantize_residual")
    return codes, scales


def gemm(A, B, swap_ab: bool = False, stream=None):
    """D = A @ B.T on the tcgen05 kernel; A [m,k], B [n,k] bf16 (cuda); returns fp32 [m,n]."""
    import torch
    m, k = A.shape
    n = B.shape[0]
    D = torch.empty((m, n), dtype=torch.float32, device=A.device)
    nb = int(lib().fl_test_gemm_scratch_bytes(m, n, k, int(swap_ab)))
    scratch = torch.empty(max(nb, 256) + 256, dtype=torch.uint8, device=A.device)
    sp = scratch.data_ptr() + ((-scratch.data_ptr()) % 256)
    _check(lib().fl_test_gemm(_ptr(A), _ptr(B), _ptr(D), m, n, k, int(swap_ab), ctypes.c_void_p(sp), nb,
                              _stream_ptr(stream)), "fl_test_gemm")
    return D


def gemm_noalloc(A, B, out=None, stream=None):
    """D = A @ B.T (m <= 64) through the entry point that allocates nothing:
    its split-K scratch is an array inside the library.  ``out`` (fp32 [m, n])
    may be given so the call itself allocates nothing on the torch side either."""
    import torch
    m, k = A.shape
    n = B.shape[0]
    D = out if out is not None else torch.empty((m, n), dtype=torch.float32, device=A.device)
    _check(lib().fl_gemm_skinny_noalloc(_ptr(A), _ptr(B), _ptr(D), m, n, k, _stream_ptr(stream)),
           "fl_gemm_skinny_noalloc")
    return D
