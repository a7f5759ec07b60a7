"""Python binding of libstqmoe.so (ctypes): argument marshalling only.

Every function here takes torch tensors that already live on the GPU, checks
their dtype/shape on the host, and passes raw device pointers and sizes to the C
ABI declared in include/stqmoe.h.  All arithmetic happens in the CUDA kernels of
the library; there is no CPU fallback.  If the shared library is missing or
cannot be loaded, importing this package raises.

STQMOE_CHECKED=1 in the environment loads the checked build (libstqmoe_checked.so,
`build.py --checked`): same ABI, with device-side re-checks of data-derived indices.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
CHECKED = os.environ.get("STQMOE_CHECKED", "0") == "1"
LIB_PATH = os.path.join(_HERE, "libstqmoe_checked.so" if CHECKED else "libstqmoe.so")

STQ_OK = 0
STATUS = {
    0: "STQ_OK", -1: "STQ_ERR_INVALID_ARG", -2: "STQ_ERR_SHAPE", -3: "STQ_ERR_ALIGN",
    -4: "STQ_ERR_NONFINITE", -5: "STQ_ERR_CUDA", -6: "STQ_ERR_DEVICE", -7: "STQ_ERR_WORKSPACE",
    -8: "STQ_ERR_TIMEOUT", -9: "STQ_ERR_UNSUPPORTED",
}
FMT_STQ1_0 = 0
FMT_MXFP4 = 1

# Every symbol include/stqmoe.h declares, with (restype, argtypes).
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


class MoeDesc(ctypes.Structure):
    _fields_ = [("T", _i32), ("H", _i32), ("I", _i32), ("E", _i32), ("k", _i32),
                ("out_fp32", _i32), ("add_residual", _i32), ("regime", _i32), ("norm_out", _i32),
                ("norm_eps", ctypes.c_float)]


class MoeWeights(ctypes.Structure):
    _fields_ = [("fmt", _i32), ("gate", _vp), ("up", _vp), ("down", _vp),
                ("gate_sc", _vp), ("up_sc", _vp), ("down_sc", _vp),
                ("sh_gate", _vp), ("sh_up", _vp), ("sh_down", _vp),
                ("sh_fmt", _i32), ("sh_gate_sc", _vp), ("sh_up_sc", _vp), ("sh_down_sc", _vp)]


SIGNATURES = {
    "stq_status_string": (ctypes.c_char_p, [_i32]),
    "stq_abi_version": (_i32, []),
    "stq_kernel_kind_name": (ctypes.c_char_p, [_i32]),
    "stq_checked_build": (_i32, []),
    "stq_read_error": (_i32, [_vp, _vp]),
    "stq1_pack": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "stq1_unpack": (_i32, [_vp, _i64, _i64, _vp, _vp]),
    "stq1_pack_ls": (_i32, [_vp, _vp, _i64, _i64, _vp, _vp, _vp]),
    "mxfp4_pack": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "mxfp4_unpack": (_i32, [_vp, _vp, _i64, _i64, _vp, _vp]),
    "mxfp8_quantize_bf16": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "stq1_gemv": (_i32, [_vp, _i64, _i64, _vp, _i64, _vp, _vp]),
    "w4a8_gemm": (_i32, [_vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp]),
    "moe_router_topk": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp]),
    "stq_router_ksplit": (_i32, [_i32]),
    "moe_router_topk_static": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_permute": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_workspace_bytes": (_sz, [ctypes.POINTER(MoeDesc)]),
    "moe_workspace_offset": (_sz, [ctypes.POINTER(MoeDesc), _i32]),
    "moe_expert_forward": (_i32, [ctypes.POINTER(MoeDesc), _vp, _vp, _vp, ctypes.POINTER(MoeWeights),
                                  _vp, _vp, _sz, _vp]),
    "moe_get_device_error": (_i32, [_vp, _vp]),
    "stq_set_timing": (_i32, [_vp]),
    "stq_wait_selftest": (_i32, [_vp, _vp]),
    "stq_slot_bank_create": (_vp, [_i32, _i32]),
    "stq_slot_bank_destroy": (None, [_vp]),
    "stq_slot_bank_map": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _vp]),
    "stq_slot_bank_resident": (_i32, [_vp, _vp]),
    "stq_slot_bank_copy": (_i32, [_vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "stq_rmsnorm_bf16": (_i32, [_vp, _i64, _i64, ctypes.c_float, _vp, _vp]),
}


KERNEL_KINDS = ["router_logits", "router_topk", "permute", "quant_x", "gate_up", "down", "combine", "gemv", "gemm",
                "gate_up_mx", "down_mx", "plan", "shared_gate_up", "shared_down", "rmsnorm",
                "pack_ls", "gate_up_stq_tc", "down_stq_tc", "act_limbs"]


class StqTiming(ctypes.Structure):
    _fields_ = [("events", ctypes.POINTER(ctypes.c_void_p)), ("capacity", _i32), ("kinds", ctypes.POINTER(_i32)),
                ("count", _i32)]


class KernelTimer:
    """Installs the library's timing hook: each kernel launched outside stream
    capture is bracketed by CUDA events on its own stream."""

    def __init__(self, capacity=512):
        self.cap = capacity
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.ev:          # torch creates the CUDA event on first record
            e.record()
        torch.cuda.synchronize()
        self._evp = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.ev])
        self._kinds = (_i32 * capacity)()
        self.st = StqTiming(ctypes.cast(self._evp, ctypes.POINTER(ctypes.c_void_p)), capacity,
                            ctypes.cast(self._kinds, ctypes.POINTER(_i32)), 0)

    def __enter__(self):
        self.st.count = 0
        lib.stq_set_timing(ctypes.byref(self.st))
        return self

    def __exit__(self, *a):
        lib.stq_set_timing(None)

    def results(self):
        """[(kind name, milliseconds)] for the recorded launches (synchronises)."""
        torch.cuda.synchronize()
        return [(KERNEL_KINDS[self._kinds[i]], self.ev[2 * i].elapsed_time(self.ev[2 * i + 1]))
                for i in range(self.st.count)]


def _load():
    if not os.path.exists(LIB_PATH):
        how = " --checked" if CHECKED else ""
        raise ImportError(f"{LIB_PATH} is missing: build it with `python bit_quantized_moe_stq1_b200/build.py{how}`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class StqError(RuntimeError):
    def __init__(self, status, what):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


def _check(status, what):
    if status != STQ_OK:
        raise StqError(status, what)
    return status


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


# ----------------------------------------------------------------------------- formats


def stq1_packed_bytes(rows, K):
    return rows * (K // 256) * 42


def stq1_pack(w, out=None, err=None, stream=None):
    """float32 [rows, K] -> uint8 [rows*K/256*42] (STQ1_0 layout of include/stqmoe.h)."""
    _dev(w)
    assert w.dtype == torch.float32 and w.dim() == 2
    rows, K = w.shape
    if out is None:
        out = torch.empty(stq1_packed_bytes(rows, K), dtype=torch.uint8, device=w.device)
    _check(lib.stq1_pack(_ptr(w), rows, K, _ptr(out), _ptr(err), _stream(stream)), "stq1_pack")
    return out


def stq1_pack_ls(w, importance=None, out=None, err=None, stream=None):
    """float32 [rows, K] -> STQ1_0 bytes by the least-squares encoder; importance:
    float32 [K] column weights (None = all 1)."""
    _dev(w)
    assert w.dtype == torch.float32 and w.dim() == 2
    rows, K = w.shape
    if importance is not None:
        assert importance.dtype == torch.float32 and importance.shape == (K,) and importance.is_contiguous()
    if out is None:
        out = torch.empty(stq1_packed_bytes(rows, K), dtype=torch.uint8, device=w.device)
    imp = _ptr(importance) if importance is not None else None
    _check(lib.stq1_pack_ls(_ptr(w), imp, rows, K, _ptr(out), _ptr(err), _stream(stream)), "stq1_pack_ls")
    return out


def stq1_unpack(packed, rows, K, out=None, stream=None):
    _dev(packed)
    if out is None:
        out = torch.empty((rows, K), dtype=torch.float32, device=packed.device)
    _check(lib.stq1_unpack(_ptr(packed), rows, K, _ptr(out), _stream(stream)), "stq1_unpack")
    return out


def mxfp4_pack(w, err=None, stream=None):
    _dev(w)
    assert w.dtype == torch.float32 and w.dim() == 2
    rows, K = w.shape
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((rows, K // 32), dtype=torch.uint8, device=w.device)
    _check(lib.mxfp4_pack(_ptr(w), rows, K, _ptr(codes), _ptr(scales), _ptr(err), _stream(stream)), "mxfp4_pack")
    return codes, scales


def mxfp4_unpack(codes, scales, rows, K, stream=None):
    _dev(codes, scales)
    out = torch.empty((rows, K), dtype=torch.float32, device=codes.device)
    _check(lib.mxfp4_unpack(_ptr(codes), _ptr(scales), rows, K, _ptr(out), _stream(stream)), "mxfp4_unpack")
    return out


def mxfp8_quantize_bf16(x, codes=None, scales=None, stream=None):
    """bf16 [rows, K] -> (uint8 codes [rows, K], uint8 scales [rows, K/32])."""
    _dev(x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    rows, K = x.shape
    if codes is None:
        codes = torch.empty((rows, K), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows, K // 32), dtype=torch.uint8, device=x.device)
    _check(lib.mxfp8_quantize_bf16(_ptr(x), rows, K, _ptr(codes), _ptr(scales), _stream(stream)),
           "mxfp8_quantize_bf16")
    return codes, scales


def rmsnorm_bf16(x, eps=1e-6, y=None, stream=None):
    """bf16 [T, H] -> bf16 [T, H]: each row times 1/sqrt(mean(row^2) + eps); y may be x."""
    _dev(x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    if y is None:
        y = torch.empty_like(x)
    _check(lib.stq_rmsnorm_bf16(_ptr(x), x.shape[0], x.shape[1], float(eps), _ptr(y), _stream(stream)),
           "stq_rmsnorm_bf16")
    return y


def wait_selftest(err, stream=None):
    """Run the bounded-wait self-test (about two seconds); *err then holds STQ_ERR_TIMEOUT."""
    _check(lib.stq_wait_selftest(_ptr(err), _stream(stream)), "stq_wait_selftest")


def read_error(err, stream=None):
    return lib.stq_read_error(_ptr(err), _stream(stream))


# ----------------------------------------------------------------------------- products


def stq1_gemv(W, rows, K, x, y=None, stream=None):
    """y [n, rows] float32 = x [n, K] (bf16) times the STQ1_0 matrix W [rows, K]."""
    _dev(W, x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.shape[1] == K
    n = x.shape[0]
    if y is None:
        y = torch.empty((n, rows), dtype=torch.float32, device=x.device)
    _check(lib.stq1_gemv(_ptr(W), rows, K, _ptr(x), n, _ptr(y), _stream(stream)), "stq1_gemv")
    return y


def w4a8_gemm(w_codes, w_scales, N, K, a_codes, a_scales, y=None, err=None, stream=None):
    """y [M, N] float32 = MXFP8 activations [M, K] times MXFP4 weights [N, K]^T."""
    _dev(w_codes, w_scales, a_codes, a_scales)
    M = a_codes.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=a_codes.device)
    _check(lib.w4a8_gemm(_ptr(w_codes), _ptr(w_scales), N, K, _ptr(a_codes), _ptr(a_scales), M, _ptr(y),
                         _ptr(err), _stream(stream)), "w4a8_gemm")
    return y


# ----------------------------------------------------------------------------- MoE layer


def moe_router_topk(x, w_router, k, logits=None, ids=None, w=None, stream=None):
    _dev(x, w_router)
    T, H = x.shape
    E = w_router.shape[0]
    dev = x.device
    ks = lib.stq_router_ksplit(H)
    logits = logits if logits is not None else torch.empty((ks * T, E), dtype=torch.float32, device=dev)
    ids = ids if ids is not None else torch.empty((T, k), dtype=torch.int32, device=dev)
    w = w if w is not None else torch.empty((T, k), dtype=torch.float32, device=dev)
    _check(lib.moe_router_topk(_ptr(x), _ptr(w_router), T, H, E, k, _ptr(logits), _ptr(ids), _ptr(w),
                               _stream(stream)), "moe_router_topk")
    return ids, w, logits[:T]


def moe_router_topk_static(x, w_router, k, ids=None, w=None, stream=None):
    """Router whose logits scratch is the library's own fixed per-GPU array (no
    scratch argument; see moe_router_topk_static in include/stqmoe.h)."""
    _dev(x, w_router)
    T, H = x.shape
    E = w_router.shape[0]
    ids = ids if ids is not None else torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = w if w is not None else torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(lib.moe_router_topk_static(_ptr(x), _ptr(w_router), T, H, E, k, _ptr(ids), _ptr(w), _stream(stream)),
           "moe_router_topk_static")
    return ids, w


def router_scratch(T, H, E, device):
    """Logits scratch of the router: stq_router_ksplit(H) * T rows of E floats."""
    return torch.empty((lib.stq_router_ksplit(H) * T, E), dtype=torch.float32, device=device)


def moe_permute(topk_ids, E, err=None, stream=None):
    """ids int32 [T, k] -> dict(counts, offsets, perm, inv, tlist, ntouched) (int32 device tensors)."""
    _dev(topk_ids)
    T, k = topk_ids.shape
    dev = topk_ids.device
    P = T * k
    out = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               perm=torch.empty(max(P, 1), dtype=torch.int32, device=dev),
               inv=torch.empty(max(P, 1), dtype=torch.int32, device=dev),
               tlist=torch.empty(E, dtype=torch.int32, device=dev),
               ntouched=torch.empty(1, dtype=torch.int32, device=dev))
    _check(lib.moe_permute(_ptr(topk_ids), T, k, E, _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["perm"]),
                           _ptr(out["inv"]), _ptr(out["tlist"]), _ptr(out["ntouched"]), _ptr(err),
                           _stream(stream)), "moe_permute")
    out["perm"], out["inv"] = out["perm"][:P], out["inv"][:P]
    return out


REGIME_AUTO, REGIME_DECODE, REGIME_PREFILL = 0, 1, 2


def make_desc(T, H, I, E, k, out_fp32=False, add_residual=False, regime=REGIME_AUTO, norm_eps=None):
    """norm_eps: None, or the eps of an RMS normalisation of the output rows (bf16 output)."""
    return MoeDesc(T, H, I, E, k, int(bool(out_fp32)), int(bool(add_residual)), int(regime),
                   int(norm_eps is not None), float(norm_eps if norm_eps is not None else 0.0))


def moe_workspace_bytes(desc):
    return int(lib.moe_workspace_bytes(ctypes.byref(desc)))


WS_REGIONS = ["counts", "offsets", "perm", "inv", "tlist", "ntouched", "h", "Y", "xq", "xs", "hq", "hs"]


def moe_workspace_view(desc, workspace, region, dtype, shape):
    """A tensor view of one workspace region (see moe_workspace_offset in include/stqmoe.h)."""
    off = int(lib.moe_workspace_offset(ctypes.byref(desc), WS_REGIONS.index(region)))
    n = 1
    for s_ in shape:
        n *= s_
    esz = torch.empty((), dtype=dtype).element_size()
    return workspace[off: off + n * esz].view(dtype).view(*shape)


SHARED_BF16, SHARED_MXFP8 = 0, 1


class ExpertWeights:
    """Device tensors of one layer's experts (kept alive by this object).  The shared
    expert is BF16 (sh_fmt SHARED_BF16) or MXFP8 (SHARED_MXFP8: sh_* E4M3 codes and
    sh_*_sc UE8M0 scales, as mxfp8_quantize_bf16 writes them)."""

    def __init__(self, fmt, gate, up, down, gate_sc=None, up_sc=None, down_sc=None,
                 sh_gate=None, sh_up=None, sh_down=None, sh_fmt=SHARED_BF16,
                 sh_gate_sc=None, sh_up_sc=None, sh_down_sc=None):
        self.fmt, self.gate, self.up, self.down = fmt, gate, up, down
        self.gate_sc, self.up_sc, self.down_sc = gate_sc, up_sc, down_sc
        self.sh_gate, self.sh_up, self.sh_down = sh_gate, sh_up, sh_down
        self.sh_fmt = sh_fmt
        self.sh_gate_sc, self.sh_up_sc, self.sh_down_sc = sh_gate_sc, sh_up_sc, sh_down_sc

    def struct(self):
        return MoeWeights(self.fmt, _ptr(self.gate), _ptr(self.up), _ptr(self.down),
                          _ptr(self.gate_sc), _ptr(self.up_sc), _ptr(self.down_sc),
                          _ptr(self.sh_gate), _ptr(self.sh_up), _ptr(self.sh_down), int(self.sh_fmt),
                          _ptr(self.sh_gate_sc), _ptr(self.sh_up_sc), _ptr(self.sh_down_sc))


def moe_expert_forward(desc, x, topk_ids, topk_w, weights, y, workspace, stream=None):
    _dev(x, topk_ids, topk_w, y, workspace)
    ws = weights.struct()
    _check(lib.moe_expert_forward(ctypes.byref(desc), _ptr(x), _ptr(topk_ids), _ptr(topk_w), ctypes.byref(ws),
                                  _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream)), "moe_expert_forward")
    return y


def moe_get_device_error(workspace, stream=None):
    return lib.moe_get_device_error(_ptr(workspace), _stream(stream))


def status_string(s):
    return lib.stq_status_string(s).decode()


class SlotBank:
    """Host-side expert slot bank (see stq_slot_bank_* in include/stqmoe.h): maps each
    call's routed ids to slots and lists the experts to copy in."""

    def __init__(self, n_experts, n_slots):
        self.n_experts, self.n_slots = int(n_experts), int(n_slots)
        # kept on the instance: module globals may already be gone when a bank is
        # collected at interpreter exit
        self._destroy = lib.stq_slot_bank_destroy
        self._h = lib.stq_slot_bank_create(self.n_experts, self.n_slots)
        if not self._h:
            raise StqError(-1, "stq_slot_bank_create")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._destroy(h)
            self._h = None

    def map(self, ids):
        """ids: host int32 array-like (any shape) -> (slot ids of the same shape, experts to
        load, their slots), all numpy int32."""
        import numpy as np

        a = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
        slots = np.empty_like(a)
        le = np.empty(self.n_slots, dtype=np.int32)
        ls = np.empty(self.n_slots, dtype=np.int32)
        n = ctypes.c_int32(0)
        _check(lib.stq_slot_bank_map(self._h, a.ctypes.data, a.size, slots.ctypes.data, le.ctypes.data,
                                     ls.ctypes.data, ctypes.byref(n)), "stq_slot_bank_map")
        return slots, le[:n.value].copy(), ls[:n.value].copy()

    def resident(self):
        import numpy as np

        out = np.empty(self.n_slots, dtype=np.int32)
        _check(lib.stq_slot_bank_resident(self._h, out.ctypes.data), "stq_slot_bank_resident")
        return out

    def copy(self, load_expert, load_slot, src, dst, stream=None):
        """Copy experts into slots: src / dst are lists of contiguous expert-major tensors, one
        per matrix: src[m] [n_experts, ...] (host, ideally pinned), dst[m] [n_slots, ...] on the
        GPU, with the same bytes per expert."""
        import numpy as np

        if len(src) != len(dst):
            raise ValueError("one destination per source matrix")
        for a, b in zip(src, dst):
            if a.shape[0] != self.n_experts or b.shape[0] != self.n_slots:
                raise ValueError("source rows must be n_experts and destination rows n_slots")
            if not (a.is_contiguous() and b.is_contiguous()) or not b.is_cuda:
                raise ValueError("contiguous sources; contiguous destinations on the GPU")
            if a[0].numel() * a.element_size() != b[0].numel() * b.element_size():
                raise ValueError("bytes per expert differ between source and destination")
        le = np.ascontiguousarray(load_expert, dtype=np.int32)
        ls = np.ascontiguousarray(load_slot, dtype=np.int32)
        n_m = len(src)
        srcs = (ctypes.c_void_p * n_m)(*[t.data_ptr() for t in src])
        dsts = (ctypes.c_void_p * n_m)(*[t.data_ptr() for t in dst])
        sizes = (ctypes.c_size_t * n_m)(*[t[0].numel() * t.element_size() for t in src])
        _check(lib.stq_slot_bank_copy(self._h, le.ctypes.data, ls.ctypes.data, le.size, n_m, srcs, dsts, sizes,
                                      _stream(stream)), "stq_slot_bank_copy")
