"""Thin ctypes binding of libkvq (include/kvq.h): same names, argument marshalling only.

Every step of quantize-append, dequantize and decode attention runs in the CUDA library; this
module only converts Python/torch arguments to plain pointers and sizes.  If libkvq.so is
missing the import of any call raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvq.so")

# enums (values fixed by include/kvq.h)
FMT = {"fp16": 0, "int": 1, "nf4": 2, "ternary": 3, "sign": 4, "polar": 5, "cart": 6, "lloyd": 7, "sorted": 8}
SCALE = {"absmax": 0, "minmax": 1, "sym": 2}
ANCHOR = {"none": 0, "first_n": 1, "window": 2, "all": 3}
SIDE_K, SIDE_V = 0, 1
DOMAIN_STORED, DOMAIN_ORIGINAL = 0, 1
ERRF_CAPACITY, ERRF_SEQ_ID, ERRF_WAIT_TIMEOUT = 1, 2, 4

STATUS = {0: "KVQ_OK", -1: "KVQ_ERR_INVALID_ARG", -2: "KVQ_ERR_UNSUPPORTED", -3: "KVQ_ERR_CAPACITY",
          -4: "KVQ_ERR_CUDA", -5: "KVQ_ERR_ALLOC", -6: "KVQ_ERR_STATE"}


class kvq_side(C.Structure):
    _fields_ = [("format", C.c_int32), ("bits", C.c_int32), ("bits2", C.c_int32), ("scale_mode", C.c_int32),
                ("group", C.c_int32), ("rotation", C.c_int32), ("chan_scale", C.c_int32), ("mean_sub", C.c_int32)]


class kvq_config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("batch", C.c_int32), ("n_kv_heads", C.c_int32), ("n_q_heads", C.c_int32),
                ("head_dim", C.c_int32), ("capacity", C.c_int32), ("max_queries", C.c_int32),
                ("k", kvq_side), ("v", kvq_side), ("anchor_layer_mask", C.c_uint64), ("anchor_rule", C.c_int32),
                ("anchor_n", C.c_int32), ("sm_scale", C.c_float), ("anchor_bits", C.c_int32)]


class kvq_layout(C.Structure):
    _fields_ = [("codes", C.c_int64), ("scales", C.c_int64), ("zeros", C.c_int64), ("anchors", C.c_int64),
                ("chan_scale", C.c_int64), ("seq_len", C.c_int64), ("key_mean", C.c_int64), ("anchor_scales", C.c_int64),
                ("row_bytes", C.c_int32),
                ("n_groups", C.c_int32), ("row_stride_tokens", C.c_int32), ("anchor_rows", C.c_int32),
                ("head0", C.c_int32), ("n_heads", C.c_int32)]


EXPORTS = ["kvq_arena_bytes", "kvq_create", "kvq_arena_bytes_layers", "kvq_create_layers", "kvq_arena_bytes_heads",
           "kvq_create_heads", "kvq_free", "kvq_get_layout", "kvq_get_layout_head", "kvq_set_chan_scale", "kvq_set_seq_len",
           "kvq_quantize_append", "kvq_dequantize", "kvq_decode_attention", "kvq_decode_attention_noalloc",
           "kvq_append_decode",
           "kvq_error_flags", "kvq_nf4_levels", "kvq_lloyd_levels",
           "kvq_last_launch_count", "kvq_status_str"]

_LIB = None


def lib() -> C.CDLL:
    """Load libkvq.so (built in-tree by quantized_decode_attention_append_b200/build.py)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libkvq.so not built ({LIB_PATH}); run quantized_decode_attention_append_b200/build.py")
        L = C.CDLL(LIB_PATH)
        vp, i32, u64p = C.c_void_p, C.c_int32, C.POINTER(C.c_uint64)
        L.kvq_arena_bytes.argtypes = [C.POINTER(kvq_config), u64p]
        L.kvq_create.argtypes = [C.POINTER(kvq_config), vp, C.c_uint64, C.POINTER(vp)]
        sp = C.POINTER(kvq_side)
        L.kvq_arena_bytes_layers.argtypes = [C.POINTER(kvq_config), sp, sp, u64p]
        L.kvq_create_layers.argtypes = [C.POINTER(kvq_config), sp, sp, vp, C.c_uint64, C.POINTER(vp)]
        L.kvq_arena_bytes_heads.argtypes = [C.POINTER(kvq_config), sp, sp, u64p]
        L.kvq_create_heads.argtypes = [C.POINTER(kvq_config), sp, sp, vp, C.c_uint64, C.POINTER(vp)]
        L.kvq_get_layout_head.argtypes = [vp, i32, i32, i32, C.POINTER(kvq_layout)]
        L.kvq_free.argtypes = [vp]
        L.kvq_free.restype = None
        L.kvq_get_layout.argtypes = [vp, i32, i32, C.POINTER(kvq_layout)]
        L.kvq_set_chan_scale.argtypes = [vp, i32, vp, vp]
        L.kvq_set_seq_len.argtypes = [vp, i32, i32, vp]
        L.kvq_quantize_append.argtypes = [vp, i32, vp, vp, vp, i32, i32, vp]
        L.kvq_dequantize.argtypes = [vp, i32, i32, i32, i32, i32, vp, i32, vp]
        L.kvq_decode_attention.argtypes = [vp, i32, vp, i32, vp, vp, vp, i32, vp, vp]
        L.kvq_decode_attention_noalloc.argtypes = [vp, i32, vp, i32, vp, vp, vp, i32, vp, vp]
        L.kvq_append_decode.argtypes = [vp, i32, vp, vp, vp, i32, i32, vp, vp, i32, vp, vp]
        L.kvq_error_flags.argtypes = [vp, C.POINTER(i32)]
        L.kvq_nf4_levels.argtypes = [C.POINTER(C.c_float)]
        L.kvq_lloyd_levels.argtypes = [i32, C.POINTER(C.c_float)]
        L.kvq_last_launch_count.argtypes = [vp]
        L.kvq_last_launch_count.restype = i32
        L.kvq_status_str.argtypes = [i32]
        L.kvq_status_str.restype = C.c_char_p
        for name in EXPORTS:
            if name not in ("kvq_free", "kvq_last_launch_count", "kvq_status_str"):
                getattr(L, name).restype = i32
        _LIB = L
    return _LIB


class KVQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({kvq_status_str(status)})")


def _check(st: int, what: str):
    if st != 0:
        raise KVQError(st, what)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


# ----------------------------------------------------------------------------- config
@dataclass
class Side:
    fmt: str = "int"
    bits: int = 4
    bits2: int = 0
    scale: str = "absmax"
    group: int = 32
    rot: int = 0
    chan_scale: bool = False
    mean_sub: bool = False

    def to_c(self) -> kvq_side:
        return kvq_side(FMT[self.fmt], self.bits, self.bits2, SCALE[self.scale], self.group, self.rot,
                        1 if self.chan_scale else 0, 1 if self.mean_sub else 0)


@dataclass
class Config:
    n_layers: int
    batch: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    capacity: int
    k: Side
    v: Side
    max_queries: int = 0
    anchor_layers: tuple = ()
    anchor_rule: str = "none"
    anchor_n: int = 0
    sm_scale: float = 0.0
    layer_k: tuple = ()  # per-layer K formats (n_layers Sides); empty: k on every layer
    layer_v: tuple = ()  # per-layer V formats; empty: v on every layer
    anchor_bits: int = 16  # anchored rows as fp16 (16) or on an 8/4-bit grid in groups of 32
    head_k: tuple = ()   # per-(layer, kv-head) K formats: n_layers tuples of n_kv_heads Sides; empty: per layer
    head_v: tuple = ()   # per-(layer, kv-head) V formats

    def side(self, layer: int, side: int, head: int = 0) -> Side:
        """Format of (layer, side) for kv-head `head`."""
        ph = self.head_k if side == SIDE_K else self.head_v
        if ph:
            return ph[layer][head]
        per = self.layer_k if side == SIDE_K else self.layer_v
        return per[layer] if per else (self.k if side == SIDE_K else self.v)

    def head_arrays(self):
        """(head_k, head_v) as flat layer-major C arrays of kvq_side (every (layer, head) filled)."""
        n = self.n_layers * self.n_kv_heads
        out = []
        for sd in (SIDE_K, SIDE_V):
            arr = (kvq_side * n)(*[self.side(l, sd, h).to_c() for l in range(self.n_layers)
                                   for h in range(self.n_kv_heads)])
            out.append(arr)
        return out[0], out[1]

    def layer_arrays(self):
        """(layer_k, layer_v) as C arrays of kvq_side, or None where uniform."""
        def arr(per):
            if not per:
                return None
            assert len(per) == self.n_layers
            return (kvq_side * self.n_layers)(*[s.to_c() for s in per])
        return arr(self.layer_k), arr(self.layer_v)

    def to_c(self) -> kvq_config:
        mask = 0
        for l in self.anchor_layers:
            mask |= 1 << int(l)
        return kvq_config(self.n_layers, self.batch, self.n_kv_heads, self.n_q_heads, self.head_dim, self.capacity,
                          self.max_queries or self.batch, self.k.to_c(), self.v.to_c(), mask, ANCHOR[self.anchor_rule],
                          self.anchor_n, self.sm_scale, self.anchor_bits)


# ----------------------------------------------------------------------------- C-ABI calls
def kvq_status_str(status: int) -> str:
    return lib().kvq_status_str(status).decode()


def kvq_arena_bytes(cfg: Config) -> int:
    c = cfg.to_c()
    n = C.c_uint64(0)
    if cfg.head_k or cfg.head_v:
        hk, hv = cfg.head_arrays()
        _check(lib().kvq_arena_bytes_heads(C.byref(c), hk, hv, C.byref(n)), "kvq_arena_bytes_heads")
    elif cfg.layer_k or cfg.layer_v:
        lk, lv = cfg.layer_arrays()
        _check(lib().kvq_arena_bytes_layers(C.byref(c), lk, lv, C.byref(n)), "kvq_arena_bytes_layers")
    else:
        _check(lib().kvq_arena_bytes(C.byref(c), C.byref(n)), "kvq_arena_bytes")
    return n.value


def kvq_create(cfg: Config, arena) -> C.c_void_p:
    c = cfg.to_c()
    h = C.c_void_p()
    base, nbytes = C.c_void_p(arena.data_ptr()), arena.numel() * arena.element_size()
    if cfg.head_k or cfg.head_v:
        hk, hv = cfg.head_arrays()
        _check(lib().kvq_create_heads(C.byref(c), hk, hv, base, nbytes, C.byref(h)), "kvq_create_heads")
    elif cfg.layer_k or cfg.layer_v:
        lk, lv = cfg.layer_arrays()
        _check(lib().kvq_create_layers(C.byref(c), lk, lv, base, nbytes, C.byref(h)), "kvq_create_layers")
    else:
        _check(lib().kvq_create(C.byref(c), base, nbytes, C.byref(h)), "kvq_create")
    return h


def kvq_free(h):
    lib().kvq_free(h)


def kvq_get_layout(h, layer: int, side: int) -> kvq_layout:
    out = kvq_layout()
    _check(lib().kvq_get_layout(h, layer, side, C.byref(out)), "kvq_get_layout")
    return out


def kvq_get_layout_head(h, layer: int, side: int, head: int) -> kvq_layout:
    out = kvq_layout()
    _check(lib().kvq_get_layout_head(h, layer, side, head, C.byref(out)), "kvq_get_layout_head")
    return out


def kvq_set_chan_scale(h, layer: int, c16, stream=None):
    _check(lib().kvq_set_chan_scale(h, layer, _ptr(c16), _stream(stream)), "kvq_set_chan_scale")


def kvq_set_seq_len(h, layer: int, length: int, stream=None):
    _check(lib().kvq_set_seq_len(h, layer, length, _stream(stream)), "kvq_set_seq_len")


def kvq_quantize_append(h, layer: int, k16, v16, seq_ids, n_seqs: int, n_new: int, stream=None):
    _check(lib().kvq_quantize_append(h, layer, _ptr(k16), _ptr(v16), _ptr(seq_ids), n_seqs, n_new, _stream(stream)),
           "kvq_quantize_append")


def kvq_dequantize(h, layer: int, side: int, domain: int, t0: int, nt: int, out, stream=None):
    import torch
    fp32 = 1 if out.dtype == torch.float32 else 0
    _check(lib().kvq_dequantize(h, layer, side, domain, t0, nt, _ptr(out), fp32, _stream(stream)), "kvq_dequantize")


def kvq_decode_attention(h, layer: int, q16, n_q: int, seq_ids, kv_len, out, lse=None, stream=None):
    import torch
    fp32 = 1 if out.dtype == torch.float32 else 0
    _check(lib().kvq_decode_attention(h, layer, _ptr(q16), n_q, _ptr(seq_ids), _ptr(kv_len), _ptr(out), fp32,
                                      _ptr(lse), _stream(stream)), "kvq_decode_attention")


def kvq_decode_attention_noalloc(h, layer: int, q16, n_q: int, seq_ids, kv_len, out, lse=None, stream=None):
    """kvq_decode_attention with the split-K scratch in the library's fixed device array."""
    import torch
    fp32 = 1 if out.dtype == torch.float32 else 0
    _check(lib().kvq_decode_attention_noalloc(h, layer, _ptr(q16), n_q, _ptr(seq_ids), _ptr(kv_len), _ptr(out), fp32,
                                              _ptr(lse), _stream(stream)), "kvq_decode_attention_noalloc")


def kvq_append_decode(h, layer: int, k16, v16, seq_ids, n_seqs: int, n_new: int, q16, out, lse=None, stream=None):
    """kvq_quantize_append then kvq_decode_attention (one query per listed sequence), in one
    split-K launch where the layer allows it."""
    import torch
    fp32 = 1 if out.dtype == torch.float32 else 0
    _check(lib().kvq_append_decode(h, layer, _ptr(k16), _ptr(v16), _ptr(seq_ids), n_seqs, n_new, _ptr(q16), _ptr(out),
                                   fp32, _ptr(lse), _stream(stream)), "kvq_append_decode")


def kvq_error_flags(h) -> int:
    f = C.c_int32(0)
    _check(lib().kvq_error_flags(h, C.byref(f)), "kvq_error_flags")
    return f.value


def kvq_nf4_levels() -> list:
    arr = (C.c_float * 16)()
    _check(lib().kvq_nf4_levels(arr), "kvq_nf4_levels")
    return list(arr)


def kvq_lloyd_levels(bits: int) -> list:
    arr = (C.c_float * (1 << bits))()
    _check(lib().kvq_lloyd_levels(bits, arr), "kvq_lloyd_levels")
    return list(arr)


def kvq_last_launch_count(h) -> int:
    return lib().kvq_last_launch_count(h)


# ----------------------------------------------------------------------------- convenience
class KVCache:
    """A cache handle plus its caller-owned device arena (a torch uint8 tensor)."""

    def __init__(self, cfg: Config, device="cuda"):
        import torch
        self.cfg = cfg
        nbytes = kvq_arena_bytes(cfg)
        self.arena = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.arena.data_ptr()) % 256
        self.arena = self.arena[off:off + nbytes]
        self.h = kvq_create(cfg, self.arena)

    def close(self):
        if self.h:
            kvq_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def layout(self, layer, side, head=0):
        return kvq_get_layout_head(self.h, layer, side, head)

    def unit(self, layer: int, b: int, h: int) -> int:
        """Row of (sequence b, kv-head h) in the views of h's head group."""
        lo = self.layout(layer, SIDE_K, h)
        return b * lo.n_heads + (h - lo.head0)

    def view(self, layer: int, side: int, what: str, head: int = 0):
        """torch views into the arena regions of the head group holding kv-head `head`: codes
        [B*nh, Tcap, row_bytes] uint8, scales/zeros [B*nh, Tcap, n_groups] fp16, anchors
        [B*nh, anchor_rows, D] fp16 (or code bytes), key_mean [B*nh, D], seq_len [B] int32."""
        import torch
        lo = self.layout(layer, side, head)
        U = self.cfg.batch * lo.n_heads
        T = lo.row_stride_tokens
        if what == "codes":
            return self.arena[lo.codes:lo.codes + U * T * lo.row_bytes].view(U, T, lo.row_bytes)
        if what in ("scales", "zeros"):
            o = lo.scales if what == "scales" else lo.zeros
            if o < 0:
                return None
            n = U * T * lo.n_groups * 2
            return self.arena[o:o + n].view(torch.float16).view(U, T, lo.n_groups)
        if what == "anchors":  # fp16 rows, or code bytes for int anchors
            if lo.anchors < 0:
                return None
            D, ab = self.cfg.head_dim, self.cfg.anchor_bits
            if ab == 16:
                n = U * lo.anchor_rows * D * 2
                return self.arena[lo.anchors:lo.anchors + n].view(torch.float16).view(U, lo.anchor_rows, D)
            n = U * lo.anchor_rows * D * ab // 8
            return self.arena[lo.anchors:lo.anchors + n].view(U, lo.anchor_rows, D * ab // 8)
        if what == "anchor_scales":
            if lo.anchor_scales < 0:
                return None
            n = U * lo.anchor_rows * (self.cfg.head_dim // 32) * 2
            return self.arena[lo.anchor_scales:lo.anchor_scales + n].view(torch.float16).view(
                U, lo.anchor_rows, self.cfg.head_dim // 32)
        if what == "seq_len":
            return self.arena[lo.seq_len:lo.seq_len + 4 * self.cfg.batch].view(torch.int32)
        if what == "key_mean":
            if lo.key_mean < 0:
                return None
            n = U * self.cfg.head_dim * 2
            return self.arena[lo.key_mean:lo.key_mean + n].view(torch.float16).view(U, self.cfg.head_dim)
        raise ValueError(what)

    def set_chan_scale(self, layer, c16, stream=None):
        kvq_set_chan_scale(self.h, layer, c16, stream)

    def set_seq_len(self, layer, length, stream=None):
        kvq_set_seq_len(self.h, layer, length, stream)

    def _check_device(self, name, x):
        if x.device != self.arena.device:
            raise ValueError(f"{name}: on {x.device}, the cache arena is on {self.arena.device}")

    def _check_rows(self, name, x, n_seqs, n=None):
        """x must be a contiguous fp16 tensor [n_seqs, n_kv_heads, n, head_dim] on the arena's device."""
        import torch
        c = self.cfg
        if x.dtype != torch.float16 or not x.is_cuda or not x.is_contiguous():
            raise ValueError(f"{name}: need a contiguous fp16 CUDA tensor, got {x.dtype} on {x.device}")
        if x.dim() != 4 or tuple(x.shape[:2]) != (n_seqs, c.n_kv_heads) or x.shape[3] != c.head_dim or \
                (n is not None and x.shape[2] != n):
            raise ValueError(f"{name}: need [{n_seqs}, {c.n_kv_heads}, n, {c.head_dim}], got {tuple(x.shape)}")
        self._check_device(name, x)

    def append(self, layer, k16, v16, seq_ids=None, stream=None):
        """Append k16/v16 [n_seqs, n_kv_heads, n, head_dim] to the sequences `seq_ids` (an int32
        CUDA tensor of n_seqs distinct ids) or, with seq_ids None, to every sequence (n_seqs = batch)."""
        import torch
        n_seqs = self.cfg.batch
        if seq_ids is not None:
            if seq_ids.dtype != torch.int32 or not seq_ids.is_cuda or seq_ids.dim() != 1 or not seq_ids.is_contiguous():
                raise ValueError("seq_ids: need a contiguous 1-D int32 CUDA tensor")
            self._check_device("seq_ids", seq_ids)
            n_seqs = seq_ids.numel()
        self._check_rows("k", k16, n_seqs)
        self._check_rows("v", v16, n_seqs, k16.shape[2])
        kvq_quantize_append(self.h, layer, k16, v16, seq_ids, n_seqs, k16.shape[2], stream)

    def append_decode(self, layer, k16, v16, q16, seq_ids=None, fp32=True, lse=False, out=None, stream=None):
        """One decode step: append k16/v16 [n_seqs, n_kv_heads, n, head_dim] to the sequences
        `seq_ids` (or every sequence), then decode q16 [n_seqs, n_q_heads, head_dim], query s over
        sequence seq_ids[s]'s whole new length.  Returns out (and lse)."""
        import torch
        c = self.cfg
        n_seqs = c.batch
        if seq_ids is not None:
            if seq_ids.dtype != torch.int32 or not seq_ids.is_cuda or seq_ids.dim() != 1 or not seq_ids.is_contiguous():
                raise ValueError("seq_ids: need a contiguous 1-D int32 CUDA tensor")
            self._check_device("seq_ids", seq_ids)
            n_seqs = seq_ids.numel()
        self._check_rows("k", k16, n_seqs)
        self._check_rows("v", v16, n_seqs, k16.shape[2])
        if q16.dtype != torch.float16 or not q16.is_cuda or not q16.is_contiguous() or \
                tuple(q16.shape) != (n_seqs, c.n_q_heads, c.head_dim):
            raise ValueError(f"q: need a contiguous fp16 CUDA tensor [{n_seqs}, {c.n_q_heads}, {c.head_dim}], got "
                             f"{q16.dtype} {tuple(q16.shape)} on {q16.device}")
        self._check_device("q", q16)
        if out is None:
            out = torch.empty(n_seqs, c.n_q_heads, c.head_dim, device=q16.device,
                              dtype=torch.float32 if fp32 else torch.float16)
        elif out.dtype not in (torch.float32, torch.float16) or not out.is_cuda or not out.is_contiguous() or \
                tuple(out.shape) != (n_seqs, c.n_q_heads, c.head_dim):
            raise ValueError(f"out: need a contiguous fp32 or fp16 CUDA tensor [{n_seqs}, {c.n_q_heads}, "
                             f"{c.head_dim}], got {out.dtype} {tuple(out.shape)} on {out.device}")
        else:
            self._check_device("out", out)
        l = torch.empty(n_seqs, c.n_q_heads, device=q16.device, dtype=torch.float32) if lse else None
        kvq_append_decode(self.h, layer, k16, v16, seq_ids, n_seqs, k16.shape[2], q16, out, l, stream)
        return (out, l) if lse else out

    def dequantize(self, layer, side, t0, nt, domain=DOMAIN_STORED, fp32=True, stream=None):
        import torch
        c = self.cfg
        out = torch.empty(c.batch, c.n_kv_heads, nt, c.head_dim, device=self.arena.device,
                          dtype=torch.float32 if fp32 else torch.float16)
        kvq_dequantize(self.h, layer, side, domain, t0, nt, out, stream)
        return out

    def decode(self, layer, q16, seq_ids=None, kv_len=None, fp32=True, lse=False, out=None, stream=None):
        import torch
        c = self.cfg
        if q16.dtype != torch.float16 or not q16.is_cuda or not q16.is_contiguous() or q16.dim() != 3 or \
                tuple(q16.shape[1:]) != (c.n_q_heads, c.head_dim):
            raise ValueError(f"q: need a contiguous fp16 CUDA tensor [n_q, {c.n_q_heads}, {c.head_dim}], got "
                             f"{q16.dtype} {tuple(q16.shape)} on {q16.device}")
        self._check_device("q", q16)
        for name, t in (("seq_ids", seq_ids), ("kv_len", kv_len)):
            if t is not None and (t.dtype != torch.int32 or not t.is_cuda or t.numel() != q16.shape[0] or
                                  not t.is_contiguous()):
                raise ValueError(f"{name}: need a contiguous int32 CUDA tensor of n_q = {q16.shape[0]} entries")
            if t is not None:
                self._check_device(name, t)
        n_q = q16.shape[0]
        if out is None:
            out = torch.empty(n_q, self.cfg.n_q_heads, self.cfg.head_dim, device=q16.device,
                              dtype=torch.float32 if fp32 else torch.float16)
        elif out.dtype not in (torch.float32, torch.float16) or not out.is_cuda or not out.is_contiguous() or \
                tuple(out.shape) != (n_q, c.n_q_heads, c.head_dim):
            raise ValueError(f"out: need a contiguous fp32 or fp16 CUDA tensor [{n_q}, {c.n_q_heads}, {c.head_dim}], "
                             f"got {out.dtype} {tuple(out.shape)} on {out.device}")
        else:
            self._check_device("out", out)
        l = torch.empty(n_q, self.cfg.n_q_heads, device=q16.device, dtype=torch.float32) if lse else None
        kvq_decode_attention(self.h, layer, q16, n_q, seq_ids, kv_len, out, l, stream)
        return (out, l) if lse else out
