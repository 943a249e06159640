"""Thin ctypes binding of libsg (include/sg.h).  Argument marshalling only: every
step of the matcher runs in the library's CUDA kernels.  Torch is used for
device memory and streams; the calls take torch tensors and pass their device
pointers through the C ABI.

The library is loaded from this package directory (built in-tree by
``learned_sparse_feature_b200.build``); a missing library is an error, there is
no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsg.so")

SG_MAX_STAGES = 32
SG_ENC_LAYERS = 5

STATUS = {0: "SG_OK", 1: "SG_ERR_INVALID_ARG", 2: "SG_ERR_SHAPE", 3: "SG_ERR_OOM",
          4: "SG_ERR_CUDA", 5: "SG_ERR_TIMEOUT", 6: "SG_ERR_NUMERIC", 7: "SG_ERR_UNSUPPORTED"}

EXPORTED = ["sg_create", "sg_destroy", "sg_match", "sg_match_host", "sg_scores",
            "sg_optimal_transport", "sg_status", "sg_strerror", "sg_launches_per_match",
            "sg_selftest_barrier_timeout", "sg_profile", "sg_profile_read",
            "sg_optimal_transport_static", "sg_selftest_exp2_poly", "sg_assign_double_softmax",
            "sg_layers_run"]

KERNEL_CLASSES = ["encoder", "qkv_gemm", "attention", "mlp1_gemm", "mlp2_gemm", "proj_gemm",
                  "score_gemm", "sinkhorn", "gnn"]

_FP = C.POINTER(C.c_float)


class SgWeights(C.Structure):
    _fields_ = [
        ("enc_W", _FP * SG_ENC_LAYERS),
        ("enc_b", _FP * SG_ENC_LAYERS),
        ("enc_bn", (_FP * 4) * (SG_ENC_LAYERS - 1)),
        ("Wq", _FP * SG_MAX_STAGES), ("bq", _FP * SG_MAX_STAGES),
        ("Wk", _FP * SG_MAX_STAGES), ("bk", _FP * SG_MAX_STAGES),
        ("Wv", _FP * SG_MAX_STAGES), ("bv", _FP * SG_MAX_STAGES),
        ("Wm", _FP * SG_MAX_STAGES), ("bm", _FP * SG_MAX_STAGES),
        ("W1", _FP * SG_MAX_STAGES), ("b1", _FP * SG_MAX_STAGES),
        ("bn1", (_FP * 4) * SG_MAX_STAGES),
        ("W2", _FP * SG_MAX_STAGES),
        ("Wf", _FP), ("bf", _FP),
        ("bin_score", C.c_float),
        ("lg_Wp", _FP), ("lg_bp", _FP), ("lg_wz", _FP), ("lg_bz", C.c_float),
        ("tc_w", _FP * (SG_MAX_STAGES // 2)), ("tc_b", C.c_float * (SG_MAX_STAGES // 2)),
    ]


class SgConfig(C.Structure):
    _fields_ = [
        ("D", C.c_int), ("H", C.c_int), ("n_stages", C.c_int), ("sinkhorn_iters", C.c_int),
        ("match_threshold", C.c_float), ("bn_eps", C.c_float), ("precision", C.c_int),
        ("img_w", C.c_float), ("img_h", C.c_float), ("norm_mode", C.c_int),
        ("max_B", C.c_int), ("max_M", C.c_int), ("max_N", C.c_int),
        ("head", C.c_int),
        ("depth_confidence", C.c_float),
    ]


HEADS = {"sinkhorn": 0, "double_softmax": 1}


class SgError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


_lib = None


def load():
    """Load libsg.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libsg.so not built at {LIB_PATH}; run learned_sparse_feature_b200.build")
    lib = C.CDLL(LIB_PATH)
    vp, i32, f32 = C.c_void_p, C.c_int, C.c_float
    lib.sg_create.argtypes = [C.POINTER(SgWeights), C.POINTER(SgConfig), C.POINTER(vp)]
    lib.sg_create.restype = i32
    lib.sg_destroy.argtypes = [vp]
    lib.sg_destroy.restype = None
    io = [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.sg_match.argtypes = io + [vp, vp, vp, vp, vp, vp]
    lib.sg_match.restype = i32
    lib.sg_match_host.argtypes = io + [vp, vp, vp, vp, vp, vp]
    lib.sg_match_host.restype = i32
    lib.sg_scores.argtypes = io + [vp, vp]
    lib.sg_scores.restype = i32
    lib.sg_optimal_transport.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.sg_optimal_transport.restype = i32
    lib.sg_assign_double_softmax.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.sg_assign_double_softmax.restype = i32
    lib.sg_status.argtypes = [vp, vp]
    lib.sg_status.restype = i32
    lib.sg_strerror.argtypes = [i32]
    lib.sg_strerror.restype = C.c_char_p
    lib.sg_launches_per_match.argtypes = [vp, i32, i32, i32]
    lib.sg_launches_per_match.restype = i32
    lib.sg_selftest_barrier_timeout.argtypes = [vp, C.c_uint, vp]
    lib.sg_selftest_barrier_timeout.restype = i32
    lib.sg_profile.argtypes = [vp, i32]
    lib.sg_profile.restype = i32
    lib.sg_profile_read.argtypes = [vp, C.POINTER(C.c_float), C.POINTER(C.c_int), i32]
    lib.sg_profile_read.restype = i32
    lib.sg_optimal_transport_static.argtypes = [i32, i32, i32, vp, f32, i32, f32, vp, vp, vp, vp, vp, vp, vp]
    lib.sg_optimal_transport_static.restype = i32
    lib.sg_layers_run.argtypes = [vp, C.POINTER(C.c_int), vp]
    lib.sg_layers_run.restype = i32
    lib.sg_selftest_exp2_poly.argtypes = [vp, vp, i32, vp]
    lib.sg_selftest_exp2_poly.restype = i32
    _lib = lib
    return lib


def _check(code, where):
    if code != 0:
        raise SgError(code, where)


def _ptr(t):
    """Device (or host) pointer of a torch tensor / numpy array, or None."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream_ptr(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Matcher:
    """A libsg handle: packed weights plus a workspace for (max_B, max_M, max_N)."""

    def __init__(self, weights: dict, max_B: int, max_M: int, max_N: int, precision: str = "bf16",
                 n_stages: int | None = None, sinkhorn_iters: int = 100, match_threshold: float = 0.2,
                 bn_eps: float = 1e-5, img_w: float = 640.0, img_h: float = 480.0, norm_mode: int = 0,
                 head: str = "sinkhorn", depth_confidence: float = -1.0):
        lib = load()
        self._keep = []
        w = SgWeights()

        def fp(a):
            a = np.ascontiguousarray(np.asarray(a, np.float32))
            self._keep.append(a)
            return a.ctypes.data_as(_FP)

        for l in range(SG_ENC_LAYERS):
            w.enc_W[l] = fp(weights["enc_W"][l])
            w.enc_b[l] = fp(weights["enc_b"][l])
            if l < SG_ENC_LAYERS - 1:
                for k in range(4):
                    w.enc_bn[l][k] = fp(weights["enc_bn"][l][k])
        stages = weights["stages"]
        n = len(stages) if n_stages is None else n_stages
        for s in range(n):
            st = stages[s]
            for nm in ("Wq", "bq", "Wk", "bk", "Wv", "bv", "Wm", "bm", "W1", "b1", "W2"):
                getattr(w, nm)[s] = fp(st[nm])
            for k in range(4):
                w.bn1[s][k] = fp(st["bn1"][k])
        w.Wf = fp(weights["Wf"])
        w.bf = fp(weights["bf"])
        w.bin_score = float(weights["bin_score"])
        if head == "double_softmax":
            w.lg_Wp = fp(weights["lg_Wp"])
            w.lg_bp = fp(weights["lg_bp"])
            w.lg_wz = fp(weights["lg_wz"])
            w.lg_bz = float(weights["lg_bz"])
        if depth_confidence > 0:
            for l in range(n // 2 - 1):
                w.tc_w[l] = fp(weights["tc_w"][l])
                w.tc_b[l] = float(weights["tc_b"][l])
        cfg = SgConfig(256, 4, n, sinkhorn_iters, match_threshold, bn_eps,
                       1 if precision == "bf16" else 0, img_w, img_h, norm_mode, max_B, max_M, max_N,
                       HEADS[head], depth_confidence)
        h = C.c_void_p()
        _check(lib.sg_create(C.byref(w), C.byref(cfg), C.byref(h)), "sg_create")
        self._keep = []
        self.h = h
        self.lib = lib
        self.cfg = cfg

    def close(self):
        if getattr(self, "h", None):
            self.lib.sg_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- device API -----------------------------------------------------------------
    def match(self, kpts0, conf0, desc0, kpts1, conf1, desc1, out_logP, matches0, matches1,
              mscores0, mscores1, stream=None):
        B, M, N = kpts0.shape[0], kpts0.shape[1], kpts1.shape[1]
        _check(self.lib.sg_match(self.h, B, M, N, _ptr(kpts0), _ptr(conf0), _ptr(desc0), _ptr(kpts1),
                                 _ptr(conf1), _ptr(desc1), _ptr(out_logP), _ptr(matches0),
                                 _ptr(matches1), _ptr(mscores0), _ptr(mscores1), _stream_ptr(stream)),
               "sg_match")

    def match_host(self, kpts0, conf0, desc0, kpts1, conf1, desc1, out_logP, matches0, matches1,
                   mscores0, mscores1, stream=None):
        B, M, N = kpts0.shape[0], kpts0.shape[1], kpts1.shape[1]
        _check(self.lib.sg_match_host(self.h, B, M, N, _ptr(kpts0), _ptr(conf0), _ptr(desc0),
                                      _ptr(kpts1), _ptr(conf1), _ptr(desc1), _ptr(out_logP),
                                      _ptr(matches0), _ptr(matches1), _ptr(mscores0), _ptr(mscores1),
                                      _stream_ptr(stream)), "sg_match_host")

    def scores(self, kpts0, conf0, desc0, kpts1, conf1, desc1, out_scores, stream=None):
        B, M, N = kpts0.shape[0], kpts0.shape[1], kpts1.shape[1]
        _check(self.lib.sg_scores(self.h, B, M, N, _ptr(kpts0), _ptr(conf0), _ptr(desc0), _ptr(kpts1),
                                  _ptr(conf1), _ptr(desc1), _ptr(out_scores), _stream_ptr(stream)),
               "sg_scores")

    def optimal_transport(self, scores, out_logP, matches0, matches1, mscores0, mscores1, stream=None):
        B, M, N = scores.shape
        _check(self.lib.sg_optimal_transport(self.h, B, M, N, _ptr(scores), _ptr(out_logP),
                                             _ptr(matches0), _ptr(matches1), _ptr(mscores0),
                                             _ptr(mscores1), _stream_ptr(stream)),
               "sg_optimal_transport")

    def assign_double_softmax(self, sim, z0, z1, out_logP, matches0, matches1, mscores0, mscores1, stream=None):
        """sg_assign_double_softmax on device tensors: sim (B, M, N), z0 (B, M), z1 (B, N)."""
        B, M, N = sim.shape
        _check(self.lib.sg_assign_double_softmax(self.h, B, M, N, _ptr(sim), _ptr(z0), _ptr(z1), _ptr(out_logP),
                                                 _ptr(matches0), _ptr(matches1), _ptr(mscores0),
                                                 _ptr(mscores1), _stream_ptr(stream)),
               "sg_assign_double_softmax")

    def status(self, stream=None):
        return self.lib.sg_status(self.h, _stream_ptr(stream))

    def selftest_barrier_timeout(self, timeout_us=20000, stream=None):
        return self.lib.sg_selftest_barrier_timeout(self.h, timeout_us, _stream_ptr(stream))

    def profile(self, enable, segments: bool = False):
        """Per-kernel timing on (events before every kernel) or off; with
        segments=True only the encoder / GNN / assignment boundaries are timed."""
        mode = (2 if segments else 1) if enable else 0
        _check(self.lib.sg_profile(self.h, mode), "sg_profile")

    def profile_read(self):
        """{class: (ms, launches)} of the last sg_match (stream must be synchronised)."""
        n = len(KERNEL_CLASSES)
        ms = (C.c_float * n)()
        cnt = (C.c_int * n)()
        if self.lib.sg_profile_read(self.h, ms, cnt, n) < 0:
            raise SgError(4, "sg_profile_read")
        return {KERNEL_CLASSES[i]: (float(ms[i]), int(cnt[i])) for i in range(n)}

    def layers_run(self, stream=None):
        """(self, cross) layers the last pass ran (synchronises the stream)."""
        n = C.c_int(0)
        _check(self.lib.sg_layers_run(self.h, C.byref(n), _stream_ptr(stream)), "sg_layers_run")
        return n.value

    def launches_per_match(self, B, M, N):
        return self.lib.sg_launches_per_match(self.h, B, M, N)


def optimal_transport_static(scores, out_logP, matches0, matches1, mscores0, mscores1, status,
                             bin_score=1.0, sinkhorn_iters=100, match_threshold=0.2, stream=None):
    """sg_optimal_transport_static: transport + extraction without any device
    allocation (library-owned static scratch).  Device tensors; `status` is a
    zeroed int32 device tensor of one element that receives device-side errors."""
    lib = load()
    B, M, N = scores.shape
    _check(lib.sg_optimal_transport_static(B, M, N, _ptr(scores), float(bin_score), int(sinkhorn_iters),
                                           float(match_threshold), _ptr(out_logP), _ptr(matches0),
                                           _ptr(matches1), _ptr(mscores0), _ptr(mscores1), _ptr(status),
                                           _stream_ptr(stream)), "sg_optimal_transport_static")


def selftest_exp2_poly(x, y, stream=None):
    """sg_selftest_exp2_poly: y = 2^x (FMA-pipe exponential of the attention
    softmax) for float32 device tensors of equal size."""
    lib = load()
    n = x.numel()
    _check(lib.sg_selftest_exp2_poly(_ptr(x), _ptr(y), int(n), _stream_ptr(stream)), "sg_selftest_exp2_poly")


def match_batch(matcher: Matcher, batch: dict, with_logP: bool = True, stream=None):
    """Convenience: run sg_match on a synthetic batch (numpy) and return numpy outputs."""
    import torch
    dev = torch.device("cuda")
    t = {k: torch.from_numpy(np.ascontiguousarray(batch[k])).to(dev)
         for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}
    B, M, N = batch["kpts0"].shape[0], batch["kpts0"].shape[1], batch["kpts1"].shape[1]
    logP = torch.empty((B, M + 1, N + 1), dtype=torch.float32, device=dev) if with_logP else None
    m0 = torch.empty((B, M), dtype=torch.int32, device=dev)
    m1 = torch.empty((B, N), dtype=torch.int32, device=dev)
    s0 = torch.empty((B, M), dtype=torch.float32, device=dev)
    s1 = torch.empty((B, N), dtype=torch.float32, device=dev)
    matcher.match(t["kpts0"], t["conf0"], t["desc0"], t["kpts1"], t["conf1"], t["desc1"],
                  logP, m0, m1, s0, s1, stream)
    _check(matcher.status(stream), "device status")
    out = {"matches0": m0.cpu().numpy(), "matches1": m1.cpu().numpy(),
           "mscores0": s0.cpu().numpy(), "mscores1": s1.cpu().numpy()}
    out["log_P"] = logP.cpu().numpy() if with_logP else None
    return out
