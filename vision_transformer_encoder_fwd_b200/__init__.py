"""Python binding of libvit_b200 (the C ABI in include/vit.h and include/vit_stages.h).

Argument marshalling only: torch supplies device memory and streams; every step of the
encoder runs in the library's CUDA kernels.  If the shared library is missing or cannot be
loaded this module raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

from . import build as _build

LIB_PATH = _build.LIB_PATH

VIT_OK = 0
VIT_E_INVALID_ARG = 1
VIT_E_SHAPE = 2
VIT_E_UNSUPPORTED = 3
VIT_E_WORKSPACE = 4
VIT_E_CUDA = 5
VIT_E_DEVICE_TIMEOUT = 6
VIT_E_NONFINITE = 7
VIT_SEG_WHOLE = 0
VIT_SEG_SLIDE = 1
KERNEL_KINDS = ("im2col", "patch_gemm", "prefix", "qkv_gemm", "attention", "proj_gemm", "fc1_gemm", "fc2_gemm",
                "tap", "final_ln", "seg_norm", "seg_cos", "seg_map", "pos_resize", "head_out", "dense_gemm", "dense_aux")


class VitConfig(ctypes.Structure):
    _fields_ = [("patch", ctypes.c_int32), ("img_h", ctypes.c_int32), ("img_w", ctypes.c_int32),
                ("dim", ctypes.c_int32), ("depth", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("mlp_dim", ctypes.c_int32), ("n_registers", ctypes.c_int32), ("pos_on_cls", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("ln_eps", ctypes.c_float), ("tap_mask", ctypes.c_uint32)]


_BLOCK_FIELDS = ("ln1_w", "ln1_b", "qkv_w", "qkv_b", "proj_w", "proj_b", "ls1", "ln2_w", "ln2_b", "fc1_w",
                 "fc1_b", "fc2_w", "fc2_b", "ls2")


class VitBlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _BLOCK_FIELDS]


class VitWeights(ctypes.Structure):
    _fields_ = [("patch_w", ctypes.c_void_p), ("patch_b", ctypes.c_void_p), ("cls", ctypes.c_void_p),
                ("reg", ctypes.c_void_p), ("pos", ctypes.c_void_p), ("norm_w", ctypes.c_void_p),
                ("norm_b", ctypes.c_void_p), ("blocks", ctypes.POINTER(VitBlockWeights))]


class VitOutputs(ctypes.Structure):
    _fields_ = [("desc", ctypes.c_void_p), ("patch_tokens", ctypes.c_void_p), ("patch_fp32", ctypes.c_int32),
                ("taps", ctypes.c_void_p * 4), ("hidden", ctypes.c_void_p)]


class VitError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


_lib = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libvit_b200.so (building it first if it is absent and nvcc is available)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        _build.build()
    lib = ctypes.CDLL(p)
    P, I32, U32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
    sigs = {
        "vit_create": (I32, [ctypes.POINTER(VitConfig), ctypes.POINTER(VitWeights), ctypes.POINTER(P)]),
        "vit_workspace_size": (I32, [P, I32, ctypes.POINTER(SZ)]),
        "vit_forward": (I32, [P, P, I32, ctypes.POINTER(VitOutputs), P, SZ, P]),
        "vit_workspace_size_hw": (I32, [P, I32, I32, I32, ctypes.POINTER(SZ)]),
        "vit_forward_hw": (I32, [P, P, I32, I32, I32, ctypes.POINTER(VitOutputs), P, SZ, P]),
        "vit_set_text_head": (I32, [P, ctypes.POINTER(VitBlockWeights), I32]),
        "vit_forward_text_tokens": (I32, [P, P, I32, I32, I32, P, P, SZ, P]),
        "vit_set_dense_head": (I32, [P, ctypes.POINTER(VitDenseHeadWeights)]),
        "vit_dense_workspace_size": (I32, [P, I32, I32, I32, ctypes.POINTER(SZ)]),
        "vit_forward_dense": (I32, [P, P, I32, I32, I32, P, P, P, SZ, P]),
        "vit_host_workspace_size": (I32, [P, I32, ctypes.POINTER(SZ)]),
        "vit_forward_host": (I32, [P, P, I32, P, P, P, SZ, P]),
        "vit_forward_noalloc": (I32, [P, P, I32, ctypes.POINTER(VitOutputs), P]),
        "vit_seg_workspace_size": (I32, [P, I32, I32, I32, I32, I32, I32, ctypes.POINTER(SZ)]),
        "vit_seg_zero_shot": (I32, [P, P, I32, I32, P, I32, I32, I32, I32, P, P, P, SZ, P]),
        "vit_poll": (I32, [P, P]),
        "vit_last_launch_count": (I32, [P]),
        "vit_destroy": (None, [P]),
        "vit_status_str": (ctypes.c_char_p, [I32]),
        "vit_last_error": (ctypes.c_char_p, []),
        "vit_profile_begin": (I32, [P, I32]),
        "vit_profile_end": (I32, [P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(I32)]),
        "vit_stage_linear": (I32, [P, P, P, I32, I32, I32, I32, P, P, P]),
        "vit_stage_linear_bounded": (I32, [P, P, P, I32, I32, I32, I32, P, P, ctypes.c_uint64, P]),
        "vit_stage_attention": (I32, [P, I32, I32, I32, P, P, P]),
        "vit_stage_attention_bounded": (I32, [P, I32, I32, I32, P, P, ctypes.c_uint64, P]),
        "vit_set_wait_limit": (I32, [P, ctypes.c_uint64]),
        "vit_stage_pos_resize": (I32, [P, I32, I32, I32, I32, I32, I32, P, P]),
        "vit_stage_gelu": (I32, [P, ctypes.c_int64, P, P]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _check(fn: str, st: int) -> None:
    if st != VIT_OK:
        lib = load_library()
        raise VitError(fn, st, lib.vit_last_error().decode(errors="replace") or lib.vit_status_str(st).decode())


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream_handle(stream) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream) or None


def config_from_spec(spec, max_batch: int) -> VitConfig:
    """vit_config from a synthetic.ModelSpec-like object."""
    mask = 0
    for l in spec.taps:
        mask |= 1 << (l - 1)
    return VitConfig(spec.patch, spec.img_h, spec.img_w, spec.dim, spec.depth, spec.heads, spec.mlp, spec.registers,
                     1 if spec.pos_on_cls else 0, max_batch, float(spec.ln_eps), mask)


_DENSE_VEC_FIELDS = ("cv1_ln_w", "cv1_ln_b", "cv2_ln_w", "cv2_ln_b", "out_ln_w", "out_ln_b", "lat_b", "smooth_b",
                     "gn_w", "gn_b", "pred_b")


class VitDenseHeadWeights(ctypes.Structure):
    _fields_ = [("n_classes", ctypes.c_int32), ("width", ctypes.c_int32), ("cv1_w", ctypes.c_void_p),
                ("cv1_ln_w", ctypes.c_void_p), ("cv1_ln_b", ctypes.c_void_p), ("bn_w", ctypes.c_void_p * 6),
                ("bn_ln_w", ctypes.c_void_p * 6), ("bn_ln_b", ctypes.c_void_p * 6), ("cv2_w", ctypes.c_void_p),
                ("cv2_ln_w", ctypes.c_void_p), ("cv2_ln_b", ctypes.c_void_p), ("out_ln_w", ctypes.c_void_p),
                ("out_ln_b", ctypes.c_void_p), ("lat_w", ctypes.c_void_p), ("lat_b", ctypes.c_void_p),
                ("smooth_w", ctypes.c_void_p), ("smooth_b", ctypes.c_void_p), ("gn_w", ctypes.c_void_p),
                ("gn_b", ctypes.c_void_p), ("pred_w", ctypes.c_void_p), ("pred_b", ctypes.c_void_p)]


class VitEncoder:
    """An encoder built from bf16 weights on the current CUDA device (vit_create)."""

    def __init__(self, spec, weights: Dict[str, object], max_batch: int, device=None):
        import torch
        self.lib = load_library()
        self.spec = spec
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.device = dev

        def to_dev(t):
            return t.to(device=dev, dtype=torch.bfloat16).contiguous()

        self.w = {k: to_dev(v) for k, v in weights.items() if k != "blocks"}
        self.wb = [{k: to_dev(v) for k, v in b.items()} for b in weights["blocks"]]
        blocks = (VitBlockWeights * spec.depth)()
        for i, b in enumerate(self.wb):
            for n in _BLOCK_FIELDS:
                setattr(blocks[i], n, _ptr(b[n]))
        self._blocks = blocks
        reg = self.w["reg"] if spec.registers > 0 else None
        vw = VitWeights(_ptr(self.w["patch_w"]), _ptr(self.w["patch_b"]), _ptr(self.w["cls"]), _ptr(reg),
                        _ptr(self.w["pos"]), _ptr(self.w["norm_w"]), _ptr(self.w["norm_b"]),
                        ctypes.cast(blocks, ctypes.POINTER(VitBlockWeights)))
        self.cfg = config_from_spec(spec, max_batch)
        h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _check("vit_create", self.lib.vit_create(ctypes.byref(self.cfg), ctypes.byref(vw), ctypes.byref(h)))
        self.handle = h
        self._ws = None

    # -------------------------------------------------------------- workspace
    def workspace_size(self, batch: int, hw=None) -> int:
        n = ctypes.c_size_t()
        if hw is None or tuple(hw) == (self.spec.img_h, self.spec.img_w):
            _check("vit_workspace_size", self.lib.vit_workspace_size(self.handle, batch, ctypes.byref(n)))
        else:
            _check("vit_workspace_size_hw", self.lib.vit_workspace_size_hw(self.handle, batch, int(hw[0]), int(hw[1]),
                                                                           ctypes.byref(n)))
        return n.value

    def grid(self, hw=None):
        """Patch grid (gh, gw) of an H x W input: the stride-p convolution's floor."""
        H, W = (self.spec.img_h, self.spec.img_w) if hw is None else hw
        return H // self.spec.patch, W // self.spec.patch

    def _workspace(self, nbytes: int):
        import torch
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self._ws

    # -------------------------------------------------------------- forward
    def alloc_outputs(self, B: int, desc=True, patch=False, patch_fp32=False, taps=False, hidden=False, hw=None):
        import torch
        s, dev = self.spec, self.device
        gh, gw = self.grid(hw)
        out = {}
        if desc:
            out["desc"] = torch.empty(B, s.dim, dtype=torch.float32, device=dev)
        if patch:
            out["patch_tokens"] = torch.empty(B, gh * gw, s.dim, device=dev,
                                              dtype=torch.float32 if patch_fp32 else torch.bfloat16)
        if taps:
            out["taps"] = [torch.empty(B, s.dim, gh, gw, dtype=torch.float32, device=dev) for _ in s.taps]
        if hidden:
            out["hidden"] = torch.empty(s.depth, B, 1 + s.registers + gh * gw, s.dim, dtype=torch.float32, device=dev)
        return out

    def forward_into(self, images, outs: Dict[str, object], stream=None, ws=None) -> None:
        """vit_forward (vit_forward_hw when images are not img_h x img_w) with caller-allocated
        outputs (see alloc_outputs)."""
        B, H, W = images.shape[0], images.shape[-2], images.shape[-1]
        native = (H, W) == (self.spec.img_h, self.spec.img_w)
        o = VitOutputs()
        o.desc = _ptr(outs.get("desc"))
        pt = outs.get("patch_tokens")
        o.patch_tokens = _ptr(pt)
        o.patch_fp32 = 1 if (pt is not None and pt.element_size() == 4) else 0
        for i, t in enumerate(outs.get("taps", [])[:4]):
            o.taps[i] = _ptr(t)
        o.hidden = _ptr(outs.get("hidden"))
        need = self.workspace_size(B, (H, W))
        wsb = ws if ws is not None else self._workspace(need)
        if native:
            _check("vit_forward", self.lib.vit_forward(self.handle, _ptr(images), B, ctypes.byref(o), _ptr(wsb),
                                                       wsb.numel(), _stream_handle(stream)))
        else:
            _check("vit_forward_hw", self.lib.vit_forward_hw(self.handle, _ptr(images), B, H, W, ctypes.byref(o),
                                                             _ptr(wsb), wsb.numel(), _stream_handle(stream)))

    def forward(self, images, desc=True, patch=False, patch_fp32=False, taps=False, hidden=False, stream=None):
        outs = self.alloc_outputs(images.shape[0], desc, patch, patch_fp32, taps, hidden,
                                  hw=(images.shape[-2], images.shape[-1]))
        self.forward_into(images, outs, stream)
        return outs

    def host_workspace_size(self, batch: int) -> int:
        n = ctypes.c_size_t()
        _check("vit_host_workspace_size", self.lib.vit_host_workspace_size(self.handle, batch, ctypes.byref(n)))
        return n.value

    def forward_host(self, images_host, desc_host, patch_host=None, stream=None, ws=None) -> None:
        """vit_forward_host: host fp32 images in, host fp32 descriptor (and bf16 patch tokens) out."""
        B = images_host.shape[0]
        need = self.host_workspace_size(B)
        wsb = ws if ws is not None else self._workspace(need)
        _check("vit_forward_host", self.lib.vit_forward_host(
            self.handle, _ptr(images_host), B, _ptr(desc_host), _ptr(patch_host), _ptr(wsb), wsb.numel(),
            _stream_handle(stream)))

    # -------------------------------------------------------------- dino.txt vision head
    def set_text_head(self, head_blocks) -> None:
        """vit_set_text_head: attach the dino.txt vision head (list of per-block bf16 weight dicts)."""
        import torch
        self.head_w = [{k: v.to(device=self.device, dtype=torch.bfloat16).contiguous() for k, v in b.items()}
                       for b in head_blocks]
        arr = (VitBlockWeights * len(self.head_w))()
        for i, b in enumerate(self.head_w):
            for n in _BLOCK_FIELDS:
                setattr(arr[i], n, _ptr(b[n]))
        self._head_arr = arr
        with torch.cuda.device(self.device):
            _check("vit_set_text_head", self.lib.vit_set_text_head(self.handle, arr, len(self.head_w)))

    def text_tokens(self, images, stream=None):
        """vit_forward_text_tokens: backbone + head -> fp32 patch tokens [B, gh*gw, D]."""
        import torch
        B, H, W = images.shape[0], images.shape[-2], images.shape[-1]
        gh, gw = self.grid((H, W))
        tok = torch.empty(B, gh * gw, self.spec.dim, dtype=torch.float32, device=self.device)
        need = self.workspace_size(B, (H, W))
        wsb = self._workspace(need)
        _check("vit_forward_text_tokens", self.lib.vit_forward_text_tokens(
            self.handle, _ptr(images), B, H, W, _ptr(tok), _ptr(wsb), wsb.numel(), _stream_handle(stream)))
        return tok

    # -------------------------------------------------------------- dense head on the taps
    def set_dense_head(self, hw) -> None:
        """vit_set_dense_head: hw = dict of bf16 weights as synthetic.make_dense_head_weights gives."""
        import torch

        def dev(t):
            return t.to(device=self.device, dtype=torch.bfloat16).contiguous()
        self.dense_w = {k: ([dev(t) for t in v] if isinstance(v, list) else dev(v)) for k, v in hw.items()}
        d = self.dense_w
        st = VitDenseHeadWeights()
        st.n_classes = int(d["pred_w"].shape[0])
        st.width = int(d["cv1_w"].shape[0])
        for k in ("cv1_w", "cv2_w", "lat_w", "smooth_w", "pred_w") + _DENSE_VEC_FIELDS:
            setattr(st, k, _ptr(d[k]))
        for i in range(6):
            st.bn_w[i] = _ptr(d["bn_w"][i])
            st.bn_ln_w[i] = _ptr(d["bn_ln_w"][i])
            st.bn_ln_b[i] = _ptr(d["bn_ln_b"][i])
        self._dense_struct = st
        with torch.cuda.device(self.device):
            _check("vit_set_dense_head", self.lib.vit_set_dense_head(self.handle, ctypes.byref(st)))

    def dense_workspace_size(self, B: int, H: int, W: int) -> int:
        n = ctypes.c_size_t()
        _check("vit_dense_workspace_size", self.lib.vit_dense_workspace_size(self.handle, B, H, W, ctypes.byref(n)))
        return n.value

    def forward_dense(self, images, p4=False, stream=None):
        """vit_forward_dense: class logits [B, K, H, W] (and projector features [B, W, gh, gw])."""
        import torch
        B, H, W = images.shape[0], images.shape[-2], images.shape[-1]
        gh, gw = self.grid((H, W))
        K, Wd = int(self.dense_w["pred_w"].shape[0]), int(self.dense_w["cv1_w"].shape[0])
        logits = torch.empty(B, K, H, W, dtype=torch.float32, device=self.device)
        feats = torch.empty(B, Wd, gh, gw, dtype=torch.float32, device=self.device) if p4 else None
        wsb = self._workspace(self.dense_workspace_size(B, H, W))
        _check("vit_forward_dense", self.lib.vit_forward_dense(
            self.handle, _ptr(images), B, H, W, _ptr(logits), _ptr(feats), _ptr(wsb), wsb.numel(),
            _stream_handle(stream)))
        return logits, feats

    # -------------------------------------------------------------- zero-shot
    def seg_workspace_size(self, H, W, C, mode, side, stride) -> int:
        n = ctypes.c_size_t()
        _check("vit_seg_workspace_size", self.lib.vit_seg_workspace_size(self.handle, H, W, C, mode, side, stride,
                                                                         ctypes.byref(n)))
        return n.value

    def seg(self, image, text, mode=VIT_SEG_SLIDE, side=384, stride=192, probs=True, labels=True, stream=None):
        import torch
        _, H, W = image.shape[-3:]
        C = text.shape[0]
        p = torch.empty(C, H, W, dtype=torch.float32, device=self.device) if probs else None
        lb = torch.empty(H, W, dtype=torch.int32, device=self.device) if labels else None
        need = self.seg_workspace_size(H, W, C, mode, side, stride)
        wsb = self._workspace(need)
        _check("vit_seg_zero_shot", self.lib.vit_seg_zero_shot(
            self.handle, _ptr(image), H, W, _ptr(text), C, mode, side, stride, _ptr(p), _ptr(lb), _ptr(wsb),
            wsb.numel(), _stream_handle(stream)))
        return p, lb

    def set_wait_limit(self, ns: int) -> None:
        """vit_set_wait_limit: the limit of every pipeline wait of later launches (0: 2 s)."""
        _check("vit_set_wait_limit", self.lib.vit_set_wait_limit(self.handle, int(ns)))

    def poll(self, stream=None) -> None:
        _check("vit_poll", self.lib.vit_poll(self.handle, _stream_handle(stream)))

    def profile_begin(self, capacity: int) -> None:
        _check("vit_profile_begin", self.lib.vit_profile_begin(self.handle, capacity))

    def profile_end(self) -> Dict[str, tuple]:
        """{kind: (total_ms, launches)} for the launches since profile_begin."""
        n = len(KERNEL_KINDS)
        ms = (ctypes.c_float * n)()
        cnt = (ctypes.c_int32 * n)()
        _check("vit_profile_end", self.lib.vit_profile_end(self.handle, ms, cnt))
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_KINDS) if cnt[i] > 0}

    def last_launch_count(self) -> int:
        return int(self.lib.vit_last_launch_count(self.handle))

    def close(self) -> None:
        if getattr(self, "handle", None):
            self.lib.vit_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------ stage entry points
def stage_linear(A, W, bias, gelu: bool = False, out=None, status=None, stream=None, wait_ns: int = 0):
    """vit_stage_linear(_bounded): out = act(A W^T + bias), bf16 in/out, fp32 bias; wait_ns > 0
    sets the limit of the kernel's pipeline waits."""
    import torch
    lib = load_library()
    M, K = A.shape
    N = W.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=A.device)
    st = status if status is not None else torch.zeros(1, dtype=torch.int32, device=A.device)
    _check("vit_stage_linear", lib.vit_stage_linear_bounded(_ptr(A), _ptr(W), _ptr(bias), M, N, K, 1 if gelu else 0,
                                                            _ptr(out), _ptr(st), int(wait_ns), _stream_handle(stream)))
    return out, st


def stage_attention(qkv, heads: int, out=None, status=None, stream=None, wait_ns: int = 0):
    """vit_stage_attention(_bounded): qkv bf16 [B, T, 3 * 64 * heads] -> out bf16 [B, T, 64 * heads];
    wait_ns > 0 sets the limit of the kernel's pipeline waits."""
    import torch
    lib = load_library()
    B, T, _ = qkv.shape
    if out is None:
        out = torch.empty(B, T, heads * 64, dtype=torch.bfloat16, device=qkv.device)
    st = status if status is not None else torch.zeros(1, dtype=torch.int32, device=qkv.device)
    _check("vit_stage_attention", lib.vit_stage_attention_bounded(_ptr(qkv), B, T, heads, _ptr(out), _ptr(st),
                                                                  int(wait_ns), _stream_handle(stream)))
    return out, st


def stage_pos_resize(pos, grid0, grid, pos_on_cls: bool, stream=None):
    """vit_stage_pos_resize: fp32 pos [(cls) + gh0*gw0, D] -> [(cls) + gh*gw, D] on the device."""
    import torch
    lib = load_library()
    D = pos.shape[1]
    out = torch.empty((1 if pos_on_cls else 0) + grid[0] * grid[1], D, dtype=torch.float32, device=pos.device)
    _check("vit_stage_pos_resize", lib.vit_stage_pos_resize(_ptr(pos), grid0[0], grid0[1], grid[0], grid[1], D,
                                                            1 if pos_on_cls else 0, _ptr(out), _stream_handle(stream)))
    return out


def stage_gelu(x, stream=None):
    """vit_stage_gelu: fp32 device tensor -> GELU(x) as the FC1 epilogue computes it."""
    import torch
    lib = load_library()
    x = x.contiguous()
    y = torch.empty_like(x)
    _check("vit_stage_gelu", lib.vit_stage_gelu(_ptr(x), x.numel(), _ptr(y), _stream_handle(stream)))
    return y

