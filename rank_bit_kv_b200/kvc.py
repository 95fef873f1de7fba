"""ctypes binding of libkvc (include/kvc.h): argument marshalling only.

Every step of the decode runs in the library's CUDA kernels; this module only
builds the C structs, owns device buffers as torch tensors (PyTorch is used
for device memory and streams) and forwards calls.  There is no fallback: if
libkvc.so is missing or fails to load, every call raises.
"""

from __future__ import annotations

import ctypes as C
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvc.so")

KVC_DENSE_BF16, KVC_LOWRANK, KVC_BLOCK_SHARED, KVC_VARRATE = 0, 1, 2, 3
STATUS = {0: "KVC_OK", 1: "KVC_EINVAL", 2: "KVC_EUNSUPPORTED", 3: "KVC_ECAPACITY",
          4: "KVC_EALIGN", 5: "KVC_EWORKSPACE", 6: "KVC_ECUDA"}
BUFS = ["lk_codes", "lk_sz", "lv_codes", "lv_sz", "rk_codes", "rk_scale", "rv_codes",
        "rv_scale", "k_dense", "v_dense", "bk", "bv", "signs_k", "signs_v", "page_table",
        "offset_k", "offset_v", "rank_k", "rank_v"]
NBUF = len(BUFS)


class LayoutDesc(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "kind", "batch", "n_q_heads", "n_kv_heads", "head_dim", "max_tokens", "n_layers",
        "rank_k", "rank_v", "latent_bits", "group_size", "latent_dim", "rope", "resid_bits",
        "page_size", "n_pages", "out_bf16", "value_bits")] + [("softmax_scale", C.c_float),
                                                               ("rope_theta", C.c_double)]


class CacheDesc(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in BUFS[:15]] + [
        ("offset_k", C.c_void_p), ("offset_v", C.c_void_p), ("rank_k", C.c_void_p),
        ("rank_v", C.c_void_p), ("seq_lens", C.c_void_p), ("n_tokens", C.c_int32),
        ("layer", C.c_int32), ("status", C.c_void_p)]

# bits of the device-side status words (include/kvc.h, KVC_DEV_*)
DEV_WAIT_TIMEOUT, DEV_BAD_POS, DEV_BAD_RANK, DEV_BAD_PAGE, DEV_BAD_OFFSET = 1, 2, 4, 8, 16


class RankBits(C.Structure):
    _fields_ = [("rank", C.c_int32), ("bits", C.c_int32)]


MAX_RESID_BITS = 8   # KVC_MAX_RESID_BITS


class KvcError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib():
    """Load libkvc.so (raises if it is missing: there is no CPU fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m rank_bit_kv_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
        L.kvc_create_layout.argtypes = [C.POINTER(LayoutDesc), C.POINTER(vp)]
        L.kvc_create_layout.restype = C.c_int
        L.kvc_destroy_layout.argtypes = [vp]
        L.kvc_destroy_layout.restype = None
        L.kvc_buffer_sizes.argtypes = [vp, C.POINTER(sz)]
        L.kvc_buffer_sizes.restype = C.c_int
        L.kvc_step_bytes.argtypes = [vp, i32]
        L.kvc_step_bytes.restype = sz
        L.kvc_workspace_bytes.argtypes = [vp, i32]
        L.kvc_workspace_bytes.restype = sz
        L.kvc_decode_launches.argtypes = [vp, i32]
        L.kvc_decode_launches.restype = i32
        L.kvc_append.argtypes = [vp, C.POINTER(CacheDesc), vp, vp, vp, i32, vp, vp]
        L.kvc_append.restype = C.c_int
        L.kvc_decode_attn.argtypes = [vp, C.POINTER(CacheDesc), vp, vp, vp, sz, vp]
        L.kvc_decode_attn.restype = C.c_int
        L.kvc_decode_attn_timed.argtypes = [vp, C.POINTER(CacheDesc), vp, vp, vp, sz, vp, vp, vp]
        L.kvc_decode_attn_timed.restype = C.c_int
        L.kvc_decode_attn_static.argtypes = [vp, C.POINTER(CacheDesc), vp, vp, vp]
        L.kvc_decode_attn_static.restype = C.c_int
        L.kvc_static_error_word.argtypes = [vp, vp]
        L.kvc_static_error_word.restype = C.c_int
        dp = C.POINTER(C.c_double)
        L.kvc_rank_bit_tables.argtypes = [i32, i32, dp, C.POINTER(C.c_int64), C.POINTER(i32), i32,
                                          C.POINTER(RankBits), i32, i32, i32, C.c_double, dp, dp,
                                          dp]
        L.kvc_rank_bit_tables.restype = C.c_int
        L.kvc_allocate_rank_bits.argtypes = [i32, i32, dp, dp, C.c_double, C.POINTER(i32), dp]
        L.kvc_allocate_rank_bits.restype = C.c_int
        L.kvc_fit_workspace_bytes.argtypes = [i32]
        L.kvc_fit_workspace_bytes.restype = sz
        L.kvc_fit_factors.argtypes = [vp, i32, i32, i32, i32, i32, vp, i32, i32, i32, vp, vp, vp,
                                      sz, vp]
        L.kvc_fit_factors.restype = C.c_int
        L.kvc_salience_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.kvc_salience_workspace_bytes.restype = sz
        L.kvc_window_salience.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, C.c_float,
                                          vp, vp, sz, vp]
        L.kvc_window_salience.restype = C.c_int
        L.kvc_ranks_by_salience.argtypes = [vp, i32, i32, i32, C.POINTER(i32), C.POINTER(i32), vp,
                                            vp]
        L.kvc_ranks_by_salience.restype = C.c_int
        L.kvc_block_keep.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
        L.kvc_block_keep.restype = C.c_int
        L.kvc_block_compact.argtypes = [vp, C.POINTER(CacheDesc), vp, C.POINTER(CacheDesc), vp,
                                        i32, vp]
        L.kvc_block_compact.restype = C.c_int
        L.kvc_select_rope_kernel.argtypes = [i32]
        L.kvc_select_rope_kernel.restype = None
        L.kvc_select_varrate_kernel.argtypes = [i32]
        L.kvc_select_varrate_kernel.restype = None
        L.kvc_test_skip_tile_copies.argtypes = [i32]
        L.kvc_test_skip_tile_copies.restype = None
        L.kvc_last_error.argtypes = []
        L.kvc_last_error.restype = C.c_char_p
        L.kvc_version.argtypes = []
        L.kvc_version.restype = C.c_char_p
        _lib = L
    return _lib


def check(status):
    if status != 0:
        raise KvcError(status, lib().kvc_last_error().decode())


def make_desc(kind, **kw):
    d = LayoutDesc()
    d.kind = {"dense": KVC_DENSE_BF16, "lowrank": KVC_LOWRANK, "block_shared": KVC_BLOCK_SHARED,
              "varrate": KVC_VARRATE}.get(kind, kind)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def desc_from_config(c, capacity=None, out_bf16=0):
    """Layout description for a synthetic-workload config dict (see synth.CONFIGS)."""
    cap = capacity or c["T"]
    kind = c["kind"]
    if kind == "lowrank":
        P = c["page"]
        if P:
            cap = -(-cap // P) * P
        return make_desc("lowrank", batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"],
                         head_dim=c["d"], max_tokens=cap, rank_k=c["rk"], rank_v=c["rv"],
                         latent_bits=c["bits"], group_size=c["g"], rope=c.get("rope", 0),
                         rope_theta=c.get("theta", 0.0), resid_bits=c["resid"], page_size=P,
                         n_pages=(c["B"] * cap // P) if P else 0, out_bf16=out_bf16)
    if kind == "varrate":
        return make_desc("varrate", batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"],
                         head_dim=c["d"], max_tokens=cap, rank_k=64, rank_v=64, latent_bits=4,
                         group_size=32, out_bf16=out_bf16)
    if kind == "block_shared":
        return make_desc("block_shared", batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"],
                         head_dim=c["d"], max_tokens=cap, n_layers=c["L"], latent_dim=c["D"],
                         group_size=c["g"], latent_bits=c.get("bits", 4),
                         value_bits=c.get("vbits", 0), out_bf16=out_bf16)
    if kind == "dense":
        return make_desc("dense", batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"],
                         head_dim=c["d"], max_tokens=cap, n_layers=c.get("L", 1),
                         out_bf16=out_bf16)
    raise ValueError(kind)


class Layout:
    """Owns a kvc_layout handle."""

    def __init__(self, desc: LayoutDesc):
        h = C.c_void_p()
        check(lib().kvc_create_layout(C.byref(desc), C.byref(h)))
        self.h = h
        self.desc = desc

    def __del__(self):
        if getattr(self, "h", None) and _lib is not None:
            _lib.kvc_destroy_layout(self.h)
            self.h = None

    def buffer_sizes(self):
        arr = (C.c_size_t * NBUF)()
        check(lib().kvc_buffer_sizes(self.h, arr))
        return dict(zip(BUFS, list(arr)))

    def workspace_bytes(self, n_tokens):
        return int(lib().kvc_workspace_bytes(self.h, n_tokens))

    def step_bytes(self, n_tokens):
        return int(lib().kvc_step_bytes(self.h, n_tokens))

    def decode_launches(self, n_tokens):
        return int(lib().kvc_decode_launches(self.h, n_tokens))


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


class Cache:
    """Device buffers of a cache (torch uint8 tensors sized by kvc_buffer_sizes)."""

    def __init__(self, layout: Layout, device="cuda", fill=None):
        import torch

        self.layout = layout
        self.bufs = {}
        for name, nbytes in layout.buffer_sizes().items():
            if nbytes:
                self.bufs[name] = torch.zeros(int(nbytes), dtype=torch.uint8, device=device)
        self.n_tokens = 0
        self.seq_lens = None
        self.status = None        # optional device int32 [1] for append's KVC_DEV_* bits
        self.layer = 0            # block-shared / layered dense: 0 all layers, l + 1 layer l
        if fill:
            self.upload(fill)

    def upload(self, arrays):
        """Copy numpy arrays (storage layout) into the matching buffers."""
        import torch

        for name, t in self.bufs.items():
            key = {"lk_codes": ("lk_codes", "kstream"), "lv_codes": ("lv_codes", "vstream"),
                   "bk": ("bk", "wk"), "bv": ("bv", "wv")}.get(name, (name,))
            a = next((arrays[k] for k in key if k in arrays), None)
            if a is None:
                continue
            raw = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
            if raw.size > t.numel():
                raise ValueError(f"{name}: {raw.size} bytes > buffer {t.numel()}")
            t[: raw.size].copy_(torch.from_numpy(raw.copy()))

    def struct(self):
        c = CacheDesc()
        for name, t in self.bufs.items():
            setattr(c, name, t.data_ptr())
        c.seq_lens = None if self.seq_lens is None else self.seq_lens.data_ptr()
        c.n_tokens = int(self.n_tokens)
        c.status = None if self.status is None else self.status.data_ptr()
        c.layer = int(self.layer)
        return c


class RawEvent:
    """A CUDA event created through the CUDA runtime that libkvc links, so that
    the library can record it (kvc_decode_attn_timed) and the caller can read
    the elapsed time."""

    _rt = None

    @classmethod
    def rt(cls):
        if cls._rt is None:
            lib()  # libkvc pulls in the CUDA runtime
            rt = C.CDLL("libcudart.so.12")
            rt.cudaEventCreate.argtypes = [C.POINTER(C.c_void_p)]
            rt.cudaEventElapsedTime.argtypes = [C.POINTER(C.c_float), C.c_void_p, C.c_void_p]
            rt.cudaEventDestroy.argtypes = [C.c_void_p]
            rt.cudaEventRecord.argtypes = [C.c_void_p, C.c_void_p]
            cls._rt = rt
        return cls._rt

    def __init__(self):
        self.cuda_event = C.c_void_p()
        err = self.rt().cudaEventCreate(C.byref(self.cuda_event))
        if err != 0:
            raise RuntimeError(f"cudaEventCreate failed ({err})")
        self.cuda_event = self.cuda_event.value

    def elapsed_ms(self, end):
        ms = C.c_float()
        err = self.rt().cudaEventElapsedTime(C.byref(ms), C.c_void_p(self.cuda_event),
                                             C.c_void_p(end.cuda_event))
        if err != 0:
            raise RuntimeError(f"cudaEventElapsedTime failed ({err})")
        return ms.value

    def record(self, stream=None):
        """Record the event on `stream` (default: torch's current stream)."""
        st = stream if stream is not None else current_stream_ptr()
        err = self.rt().cudaEventRecord(C.c_void_p(self.cuda_event), st)
        if err != 0:
            raise RuntimeError(f"cudaEventRecord failed ({err})")

    def __del__(self):
        if self._rt is not None and getattr(self, "cuda_event", None):
            self._rt.cudaEventDestroy(C.c_void_p(self.cuda_event))


def current_stream_ptr():
    import torch

    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def decode(layout: Layout, cache: Cache, q, out, ws, stream=None, events=None):
    """kvc_decode_attn on torch tensors (q bf16, out fp32/bf16, ws uint8)."""
    cs = cache.struct()
    st = stream if stream is not None else current_stream_ptr()
    if events is None:
        check(lib().kvc_decode_attn(layout.h, C.byref(cs), _ptr(q), _ptr(out), _ptr(ws),
                                    ws.numel(), st))
    else:
        check(lib().kvc_decode_attn_timed(layout.h, C.byref(cs), _ptr(q), _ptr(out), _ptr(ws),
                                          ws.numel(), st, C.c_void_p(events[0].cuda_event),
                                          C.c_void_p(events[1].cuda_event)))


STATIC_SCRATCH_BYTES = 4 << 20   # KVC_STATIC_SCRATCH_BYTES


def decode_static(layout: Layout, cache: Cache, q, out, stream=None):
    """kvc_decode_attn_static: decode with the library's built-in scratch area
    (for callers that cannot allocate a workspace)."""
    cs = cache.struct()
    st = stream if stream is not None else current_stream_ptr()
    check(lib().kvc_decode_attn_static(layout.h, C.byref(cs), _ptr(q), _ptr(out), st))


def static_error_word(dst, stream=None):
    """kvc_static_error_word: enqueue a copy of the built-in scratch area's
    error word into dst (a torch int32 tensor on the device or in pinned host
    memory)."""
    st = stream if stream is not None else current_stream_ptr()
    check(lib().kvc_static_error_word(_ptr(dst), st))


def _device_array(x, dtype, device):
    """x as a device tensor (torch tensors on the device pass through)."""
    import torch

    if isinstance(x, torch.Tensor) and x.is_cuda:
        return x
    return torch.as_tensor(np.ascontiguousarray(np.asarray(x, dtype=dtype))).to(device)


def append(layout: Layout, cache: Cache, k_new, v_new, pos, n_new, new_ranks=None,
           stream=None):
    """kvc_append: k_new / v_new torch bf16 device tensors; pos [B] and the
    VARRATE ranks [2, B, n_new] as device tensors (host sequences are copied to
    the device first)."""
    dev = k_new.device
    pos_d = _device_array(pos, np.int32, dev)
    nr_d = None if new_ranks is None else _device_array(new_ranks, np.uint8, dev)
    cs = cache.struct()
    st = stream if stream is not None else current_stream_ptr()
    check(lib().kvc_append(layout.h, C.byref(cs), _ptr(k_new), _ptr(v_new), _ptr(pos_d),
                           int(n_new), _ptr(nr_d), st))
    # keep the marshalled arrays alive until the stream has used them
    cache._append_args = (pos_d, nr_d)


# --------------------------------------------------------------------------- rank / bit allocation


def _dbl(a):
    a = np.ascontiguousarray(np.asarray(a, np.float64))
    return a, a.ctypes.data_as(C.POINTER(C.c_double))


def rank_bit_tables(spectra, rows, heads, options, head_dim, eta_latent, eta_resid,
                    latent_bits=4, group=32):
    """kvc_rank_bit_tables: (bytes, distortion) numpy [cells, options].
    options: sequence of (rank, bits); eta_resid: dict bits -> factor."""
    spectra, sp = _dbl(spectra)
    n_cells, spec_len = spectra.shape
    rows_a = np.ascontiguousarray(np.asarray(rows, np.int64))
    heads_a = np.ascontiguousarray(np.asarray(heads, np.int32))
    opts = (RankBits * len(options))(*[RankBits(int(r), int(b)) for r, b in options])
    eta = np.zeros(MAX_RESID_BITS + 1)
    for b, v in eta_resid.items():
        eta[int(b)] = v
    eta, ep = _dbl(eta)
    B = np.zeros((n_cells, len(options)))
    D = np.zeros((n_cells, len(options)))
    check(lib().kvc_rank_bit_tables(
        n_cells, spec_len, sp, rows_a.ctypes.data_as(C.POINTER(C.c_int64)),
        heads_a.ctypes.data_as(C.POINTER(C.c_int32)), len(options), opts, int(head_dim),
        int(latent_bits), int(group), float(eta_latent), ep,
        B.ctypes.data_as(C.POINTER(C.c_double)), D.ctypes.data_as(C.POINTER(C.c_double))))
    return B, D


def allocate_rank_bits(bytes_, distortion, budget):
    """kvc_allocate_rank_bits: (choice [cells] int, lambda)."""
    B, bp = _dbl(bytes_)
    D, dp = _dbl(distortion)
    n_cells, n_opt = B.shape
    ch = (C.c_int32 * n_cells)()
    lam = C.c_double()
    check(lib().kvc_allocate_rank_bits(n_cells, n_opt, bp, dp, float(budget), ch, C.byref(lam)))
    return np.array(list(ch), np.int64), lam.value


# --------------------------------------------------------------------------- factor fit


def fit_factors(x, omega, rank, power_iters, n_rows=None, stream=None, with_sigma2=True):
    """kvc_fit_factors on torch tensors: x bf16 [B, Hkv, cap, 128], omega fp32
    [Hkv, 128, k].  Returns (factor fp16 [Hkv, rank, 128], sigma2 fp32 [Hkv, k])."""
    import torch

    B, Hkv, cap, d = x.shape
    k = omega.shape[-1]
    factor = torch.empty((Hkv, rank, d), dtype=torch.float16, device=x.device)
    sigma2 = torch.empty((Hkv, k), dtype=torch.float32, device=x.device) if with_sigma2 else None
    ws = torch.empty(int(lib().kvc_fit_workspace_bytes(Hkv)), dtype=torch.uint8, device=x.device)
    st = stream if stream is not None else current_stream_ptr()
    check(lib().kvc_fit_factors(_ptr(x), B, Hkv, cap, int(n_rows or cap), d, _ptr(omega), k,
                                int(rank), int(power_iters), _ptr(factor), _ptr(sigma2),
                                _ptr(ws), ws.numel(), st))
    factor._fit_ws = ws        # keep the workspace alive until the stream has used it
    return factor, sigma2


# --------------------------------------------------------------------------- token importance


def window_salience(q_window, keys, n_tokens=None, scale=0.0, stream=None):
    """kvc_window_salience: q_window bf16 [B, Hq, W, 128], keys bf16 [B, Hkv, cap, 128]
    -> salience fp32 [B, n_tokens]."""
    import torch

    B, Hq, W, d = q_window.shape
    Hkv, cap = keys.shape[1], keys.shape[2]
    T = int(n_tokens or cap)
    sal = torch.empty((B, T), dtype=torch.float32, device=keys.device)
    ws = torch.empty(int(lib().kvc_salience_workspace_bytes(B, Hq, Hkv, W, T)),
                     dtype=torch.uint8, device=keys.device)
    st = stream if stream is not None else current_stream_ptr()
    check(lib().kvc_window_salience(_ptr(q_window), _ptr(keys), B, Hq, Hkv, W, cap, T, d,
                                    float(scale), _ptr(sal), _ptr(ws), ws.numel(), st))
    sal._ws = ws
    return sal


def ranks_by_salience(salience, rung_ranks, rung_counts, stream=None):
    """kvc_ranks_by_salience -> uint8 [2, B, T] (K ranks, V ranks)."""
    import torch

    B, T = salience.shape
    ranks = torch.empty((2, B, T), dtype=torch.uint8, device=salience.device)
    rr = (C.c_int32 * len(rung_ranks))(*[int(x) for x in rung_ranks])
    rc = (C.c_int32 * max(1, len(rung_counts)))(*[int(x) for x in rung_counts])
    st = stream if stream is not None else current_stream_ptr()
    check(lib().kvc_ranks_by_salience(_ptr(salience), B, T, len(rung_ranks), rr, rc, _ptr(ranks),
                                      st))
    return ranks


def block_keep(salience_layers, keep, stream=None):
    """kvc_block_keep: salience_layers fp32 [L, B, T] -> (importance [B, T], kept int32 [B, keep])."""
    import torch

    L, B, T = salience_layers.shape
    imp = torch.empty((B, T), dtype=torch.float32, device=salience_layers.device)
    kept = torch.empty((B, int(keep)), dtype=torch.int32, device=salience_layers.device)
    st = stream if stream is not None else current_stream_ptr()
    check(lib().kvc_block_keep(_ptr(salience_layers), L, B, T, int(keep), _ptr(imp), _ptr(kept), st))
    return imp, kept


def block_compact(src_layout, src_cache, dst_layout, dst_cache, kept, stream=None):
    """kvc_block_compact: copy the kept latent rows of src into dst."""
    a, b = src_cache.struct(), dst_cache.struct()
    st = stream if stream is not None else current_stream_ptr()
    check(lib().kvc_block_compact(src_layout.h, C.byref(a), dst_layout.h, C.byref(b), _ptr(kept),
                                  int(kept.shape[1]), st))
    dst_cache.n_tokens = int(kept.shape[1])
