"""Thin Python binding of libhpcdecode.so (C ABI declared in include/hpc_decode.h).

This module only marshals arguments. It checks tensor dtypes and devices and passes
``data_ptr()`` and the current CUDA stream to the library. Every step of the decode path
runs in the library's kernels. If the library is missing, importing this module raises
``HpcError``: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np
import torch

from .build import LIB

HPC_OK, HPC_ERR_ARG, HPC_ERR_SHAPE, HPC_ERR_DTYPE, HPC_ERR_ALIGN, HPC_ERR_CUDA, HPC_ERR_CAPACITY = range(7)
HPC_BF16, HPC_FP32, HPC_E4M3 = 0, 1, 2
HPC_HND, HPC_NHD = 0, 1
_LAYOUTS = {"HND": HPC_HND, "NHD": HPC_NHD}
DEV_STATUS = {"bad_seqlen": 0x1, "bad_page": 0x2, "capacity": 0x4, "timeout": 0x8, "bad_index": 0x10}
ITEM_DTYPE = np.dtype([("req", "<i4"), ("kv_head", "<i2"), ("flags", "<i2"),
                       ("tile_begin", "<i4"), ("tile_end", "<i4")])
ITEM_DIRECT, ITEM_SECOND_SLOT = 1, 2
RECORD_DTYPE = np.dtype([("unit_begin", "<i8"), ("unit_end", "<i8"), ("chunk", "<i8"), ("item_cost", "<i4"),
                         ("n_items", "<i4")])
ITEM_COST_DEFAULT, ITEM_COST_MAX = -1, 1024
E4M3_KERNELS = {"mma": 0, "tcgen05": 1}
MULTI_KERNELS = {"default": 0, "mma": 1, "tcgen05": 2}
TRACE_WORDS = 8
BUILD_TRACE = 1

EXPORTS = ("hpc_step_record_bytes", "hpc_build_flags", "hpc_plan_workspace_bytes", "hpc_plan_static_workspace_bytes", "hpc_decode_plan",
           "hpc_decode_plan_static", "hpc_plan_cpu", "hpc_partial_o_bytes", "hpc_partial_ml_bytes",
           "hpc_decode_attention", "hpc_merge_states", "hpc_decode_prologue", "hpc_attention_launch_info",
           "hpc_status_string", "hpc_last_error", "hpc_abi_version", "hpc_decode_step_noalloc",
           "hpc_decode_step", "hpc_decode_step_workspace_bytes", "hpc_decode_step_prologue",
           "hpc_decode_step_multi", "hpc_decode_step_multi_workspace_bytes", "hpc_decode_step_lse",
           "hpc_merge_lse", "hpc_wait_selftest", "hpc_merge_lse_gather", "hpc_gather_rows", "hpc_gather_pages")


class HpcError(RuntimeError):
    pass


class CPlan(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32), ("tile_len", ctypes.c_int32),
                ("num_ctas", ctypes.c_int32), ("max_items", ctypes.c_int32), ("merge_capacity", ctypes.c_int32),
                ("is_static", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("counts", ctypes.c_void_p), ("items", ctypes.c_void_p), ("cta_indptr", ctypes.c_void_p),
                ("merge_indptr", ctypes.c_void_p), ("merge_list", ctypes.c_void_p)]


class COptions(ctypes.Structure):
    _fields_ = [("item_cost", ctypes.c_int32), ("e4m3_kernel", ctypes.c_int32), ("record", ctypes.c_void_p),
                ("record_items", ctypes.c_int32), ("multi_kernel", ctypes.c_int32), ("trace", ctypes.c_void_p),
                ("seq_lens_ready", ctypes.c_int32)]


_path = LIB


def library_path() -> str:
    return _path


def _load(path=LIB):
    if not os.path.exists(path):
        raise HpcError(f"{path} is missing; build it with `python -m load_balanced_split_step_b200.build` "
                       "(there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    i32, vp, sz = ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
    fp = ctypes.c_float
    P = ctypes.POINTER(CPlan)
    O = ctypes.POINTER(COptions)
    sig = {
        "hpc_step_record_bytes": (sz, [i32, i32]),
        "hpc_build_flags": (ctypes.c_uint32, []),
        "hpc_plan_workspace_bytes": (sz, [i32, i32, i32]),
        "hpc_plan_static_workspace_bytes": (sz, [i32, i32, i32]),
        "hpc_decode_plan": (ctypes.c_int, [vp, i32, i32, i32, i32, i32, i32, vp, sz, P, vp, vp]),
        "hpc_decode_plan_static": (ctypes.c_int, [vp, i32, i32, i32, i32, i32, i32, vp, sz, P, vp, vp]),
        "hpc_plan_cpu": (ctypes.c_int, [vp, i32, i32, i32, i32, i32, i32, vp, sz, P, vp]),
        "hpc_partial_o_bytes": (sz, [P, i32, i32]),
        "hpc_partial_ml_bytes": (sz, [P, i32]),
        "hpc_decode_attention": (ctypes.c_int, [vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp, i32, i32, i32, i32, i32,
                                                vp, i32, vp, P, fp, vp, vp, vp, ctypes.c_int, O, vp, vp]),
        "hpc_merge_states": (ctypes.c_int, [vp, vp, P, i32, i32, vp, ctypes.c_int, vp, vp]),
        "hpc_decode_prologue": (ctypes.c_int, [vp, vp, vp, fp, fp, vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp, i32,
                                               i32, vp, i32, vp, i32, i32, i32, i32, vp, vp]),
        "hpc_attention_launch_info": (ctypes.c_int, [i32, ctypes.c_int, i32, i32, i32, i32, ctypes.POINTER(i32),
                                                     ctypes.POINTER(i32), ctypes.POINTER(i32)]),
        "hpc_decode_step_noalloc": (ctypes.c_int, [vp, vp, vp, ctypes.c_int, vp, vp, i32, i32, i32, i32, i32, vp,
                                                   i32, vp, i32, i32, i32, fp, vp, ctypes.c_int, vp, vp]),
        "hpc_decode_step_workspace_bytes": (sz, [i32, i32, i32, i32, i32]),
        "hpc_decode_step": (ctypes.c_int, [vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp, i32, i32, i32, i32, i32, vp,
                                           i32, vp, i32, i32, i32, fp, vp, sz, vp, ctypes.c_int, O, vp, vp]),
        "hpc_decode_step_prologue": (ctypes.c_int, [vp, vp, vp, fp, fp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp,
                                                    i32, i32, i32, i32, i32, vp, i32, vp, i32, i32, i32, fp, vp, sz,
                                                    vp, ctypes.c_int, O, vp, vp]),
        "hpc_decode_step_multi_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
        "hpc_decode_step_multi": (ctypes.c_int, [vp, i32, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp, i32, i32, i32,
                                                 i32, i32, vp, i32, vp, i32, i32, i32, fp, vp, sz, vp, ctypes.c_int, O,
                                                 vp, vp]),
        "hpc_decode_step_lse": (ctypes.c_int, [vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp, i32, i32, i32, i32, i32,
                                               vp, i32, vp, i32, i32, i32, fp, vp, sz, vp, ctypes.c_int, vp, O, vp, vp]),
        "hpc_merge_lse": (ctypes.c_int, [vp, vp, i32, ctypes.c_int64, i32, vp, vp, vp]),
        "hpc_wait_selftest": (ctypes.c_int, [ctypes.c_uint64, i32, vp, vp, vp]),
        "hpc_merge_lse_gather": (ctypes.c_int, [vp, vp, ctypes.c_int64, vp, i32, i32, i32, i32, vp, vp, vp, vp]),
        "hpc_gather_rows": (ctypes.c_int, [vp, ctypes.c_int64, ctypes.c_int64, vp, ctypes.c_int64, vp, vp, vp]),
        "hpc_gather_pages": (ctypes.c_int, [vp, i32, i32, vp, vp, i32, i32, vp, vp, vp]),
        "hpc_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "hpc_last_error": (ctypes.c_char_p, []),
        "hpc_abi_version": (ctypes.c_int, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib = _load()


def use_library(path: str = LIB):
    """Switch this module to another build of the library (e.g. the HPC_TRACE build, see
    ``build.build(trace=True)``); ``use_library()`` goes back to the default build."""
    global _lib, _path
    _lib = _load(path)
    _path = path


def build_flags() -> int:
    return int(_lib.hpc_build_flags())


def status_string(code: int) -> str:
    return _lib.hpc_status_string(code).decode()


def _check(rc: int, what: str):
    if rc != HPC_OK:
        raise HpcError(f"{what}: {status_string(rc)} ({rc}): {_lib.hpc_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, name, dtype=None, device=None, cuda=True):
    if not isinstance(t, torch.Tensor):
        raise HpcError(f"{name} must be a torch.Tensor")
    if cuda and not t.is_cuda:
        raise HpcError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise HpcError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise HpcError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise HpcError(f"{name} must be contiguous")


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


@dataclass
class Plan:
    """A plan bound to its workspace. ``raw`` is the C struct passed to the library."""

    raw: CPlan
    workspace: torch.Tensor
    host: bool = False

    @property
    def num_ctas(self) -> int:
        return int(self.raw.num_ctas)

    @property
    def max_items(self) -> int:
        return int(self.raw.max_items)

    def _view(self, ptr, dtype, count):
        base = self.workspace.data_ptr()
        off = int(ptr) - base
        nbytes = np.dtype(dtype).itemsize * count
        return self.workspace[off:off + nbytes]

    def to_numpy(self) -> dict:
        """Copy the plan to host: counts, the valid items, and the index arrays."""
        r = self.raw
        counts = self._view(r.counts, np.int64, 4).cpu().numpy().view(np.int64)
        n_items, n_merge = int(counts[0]), int(counts[1])
        items = self._view(r.items, ITEM_DTYPE, n_items).cpu().numpy().view(ITEM_DTYPE)
        segs = r.batch * r.kv_heads
        return {
            "n_items": n_items, "n_merge": n_merge, "n_units": int(counts[2]), "chunk": int(counts[3]),
            "items": items,
            "cta_indptr": self._view(r.cta_indptr, np.int32, r.num_ctas + 1).cpu().numpy().view(np.int32),
            "merge_indptr": self._view(r.merge_indptr, np.int32, segs + 1).cpu().numpy().view(np.int32),
            "merge_list": self._view(r.merge_list, np.int32, n_merge).cpu().numpy().view(np.int32),
        }


def plan(seq_lens: torch.Tensor, num_heads: int, kv_heads: int, tile_len: int, num_ctas: int | None = None,
         max_seq_len: int = 0, status: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> Plan:
    """Load-balanced per-step plan on the device (``hpc_decode_plan``)."""
    _need(seq_lens, "seq_lens", torch.int32)
    dev = seq_lens.device
    if num_ctas is None:
        num_ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    B = seq_lens.numel()
    nbytes = _lib.hpc_plan_workspace_bytes(B, kv_heads, num_ctas)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    raw = CPlan()
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_plan(_ptr(seq_lens), B, num_heads, kv_heads, tile_len, num_ctas, max_seq_len,
                                    _ptr(workspace), workspace.numel(), ctypes.byref(raw), _ptr(status),
                                    _stream(dev)), "hpc_decode_plan")
    return Plan(raw, workspace)


def plan_static(seq_lens: torch.Tensor, num_heads: int, kv_heads: int, tile_len: int, splits: int,
                max_seq_len: int = 0, status: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None) -> Plan:
    """Static split-k plan on the device (``hpc_decode_plan_static``)."""
    _need(seq_lens, "seq_lens", torch.int32)
    dev = seq_lens.device
    B = seq_lens.numel()
    nbytes = _lib.hpc_plan_static_workspace_bytes(B, kv_heads, splits)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    raw = CPlan()
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_plan_static(_ptr(seq_lens), B, num_heads, kv_heads, tile_len, splits, max_seq_len,
                                           _ptr(workspace), workspace.numel(), ctypes.byref(raw), _ptr(status),
                                           _stream(dev)), "hpc_decode_plan_static")
    return Plan(raw, workspace)


def plan_host(seq_lens, num_heads: int, kv_heads: int, tile_len: int, num_ctas: int,
              max_seq_len: int = 0) -> tuple[Plan, int]:
    """Host twin of ``plan`` (``hpc_plan_cpu``). Returns (plan, status word)."""
    lens = torch.as_tensor(seq_lens, dtype=torch.int32).contiguous().cpu()
    B = lens.numel()
    nbytes = _lib.hpc_plan_workspace_bytes(B, kv_heads, num_ctas)
    # 256-byte aligned host buffer
    buf = torch.empty(nbytes + 256, dtype=torch.uint8)
    off = (-buf.data_ptr()) % 256
    ws = buf[off:off + nbytes]
    st = ctypes.c_uint32(0)
    raw = CPlan()
    _check(_lib.hpc_plan_cpu(_ptr(lens), B, num_heads, kv_heads, tile_len, num_ctas, max_seq_len, _ptr(ws),
                             nbytes, ctypes.byref(raw), ctypes.byref(st)), "hpc_plan_cpu")
    p = Plan(raw, ws, host=True)
    p._keep = buf
    return p, int(st.value)


def partial_buffers(p: Plan, num_heads: int, head_dim: int, device):
    no = _lib.hpc_partial_o_bytes(ctypes.byref(p.raw), num_heads, head_dim) // 4
    nml = _lib.hpc_partial_ml_bytes(ctypes.byref(p.raw), num_heads) // 4
    return (torch.empty(max(no, 4), dtype=torch.float32, device=device),
            torch.empty(max(nml, 4), dtype=torch.float32, device=device))


_KV_DTYPES = {"bf16": HPC_BF16, "e4m3": HPC_E4M3}


def _kv_code(kv_dtype: str, t: torch.Tensor) -> int:
    if kv_dtype not in _KV_DTYPES:
        raise HpcError(f"kv_dtype must be one of {list(_KV_DTYPES)}")
    want = (torch.bfloat16,) if kv_dtype == "bf16" else (torch.uint8, torch.float8_e4m3fn)
    if t.dtype not in want:
        raise HpcError(f"cache dtype {t.dtype} does not match kv_dtype {kv_dtype}")
    return _KV_DTYPES[kv_dtype]


def _geometry(k_pages, kv_layout):
    """(num_pages, kv_heads, page_size, head_dim, layout code) of a cache tensor."""
    if kv_layout not in _LAYOUTS:
        raise HpcError(f"kv_layout must be one of {list(_LAYOUTS)}")
    if k_pages.dim() != 4:
        raise HpcError("cache must be 4-D")
    if kv_layout == "HND":
        n, hkv, psz, d = k_pages.shape
    else:
        n, psz, hkv, d = k_pages.shape
    return n, hkv, psz, d, _LAYOUTS[kv_layout]


def _cache(k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, head_dim, dev):
    """Checks the two caches against each other, the query's head_dim and the device, and the
    E4M3 scales. Returns (dtype code, num_pages, kv_heads, page_size, layout code)."""
    _need(k_pages, "k_pages", device=dev)
    _need(v_pages, "v_pages", device=dev)
    code = _kv_code(kv_dtype, k_pages)
    _kv_code(kv_dtype, v_pages)
    num_pages, Hkv, P, D, lay = _geometry(k_pages, kv_layout)
    if tuple(v_pages.shape) != tuple(k_pages.shape):
        raise HpcError(f"v_pages {tuple(v_pages.shape)} and k_pages {tuple(k_pages.shape)} differ")
    if D != head_dim:
        raise HpcError(f"cache head_dim {D} does not match the query's {head_dim}")
    if code == HPC_E4M3:
        for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
            _need(t, name, torch.float32, dev)
            if t.numel() != Hkv:
                raise HpcError(f"{name} must hold one scale per kv head ({Hkv})")
    return code, num_pages, Hkv, P, lay


def _tables(block_table, seq_lens, batch, dev):
    _need(block_table, "block_table", torch.int32, dev)
    _need(seq_lens, "seq_lens", torch.int32, dev)
    if block_table.dim() != 2 or block_table.shape[0] != batch or seq_lens.numel() != batch:
        raise HpcError(f"block_table [batch, pages] and seq_lens [batch] must match the batch of {batch}")


def _output(out, shape, out_dtype, dev):
    if out is None:
        return torch.empty(shape, dtype=out_dtype, device=dev)
    _need(out, "out", (torch.float32, torch.bfloat16), dev)
    if tuple(out.shape) != tuple(shape):
        raise HpcError(f"out has shape {tuple(out.shape)}, expected {tuple(shape)}")
    return out


def _out_code(out):
    return HPC_BF16 if out.dtype == torch.bfloat16 else HPC_FP32


def options(item_cost=None, e4m3_kernel="mma", record=None, record_items=0, trace=None, device=None, num_ctas=None,
            multi_kernel="default", seq_lens_ready=False):
    """A ``hpc_step_options`` struct, or None when every option has its default.
    item_cost: 1/16 tile per item start (None: the library's default). e4m3_kernel: "mma" or
    "tcgen05". record: uint8 device tensor of ``record_bytes(num_ctas, record_items)`` bytes.
    trace: int64 device tensor [num_ctas, TRACE_WORDS] (HPC_TRACE builds only).
    seq_lens_ready: the kernel launched just before on the stream does not write seq_lens, so the
    single-launch step may plan before waiting for it."""
    if e4m3_kernel not in E4M3_KERNELS:
        raise HpcError(f"e4m3_kernel must be one of {list(E4M3_KERNELS)}")
    if multi_kernel not in MULTI_KERNELS:
        raise HpcError(f"multi_kernel must be one of {list(MULTI_KERNELS)}")
    if (item_cost is None and e4m3_kernel == "mma" and record is None and trace is None and multi_kernel == "default"
            and not seq_lens_ready):
        return None
    o = COptions()
    o.seq_lens_ready = 1 if seq_lens_ready else 0
    o.item_cost = ITEM_COST_DEFAULT if item_cost is None else int(item_cost)
    o.e4m3_kernel = E4M3_KERNELS[e4m3_kernel]
    o.multi_kernel = MULTI_KERNELS[multi_kernel]
    if record is not None:
        _need(record, "record", torch.uint8, device)
        o.record, o.record_items = record.data_ptr(), int(record_items)
        if num_ctas is not None and record.numel() < record_bytes(num_ctas, record_items):
            raise HpcError(f"record holds {record.numel()} bytes, {record_bytes(num_ctas, record_items)} needed")
    if trace is not None:
        _need(trace, "trace", torch.int64, device)
        if num_ctas is not None and trace.numel() < num_ctas * TRACE_WORDS:
            raise HpcError(f"trace must hold num_ctas x {TRACE_WORDS} words")
        o.trace = trace.data_ptr()
    return o


def _opt_ref(o):
    return None if o is None else ctypes.byref(o)


def record_bytes(num_ctas: int, record_items: int) -> int:
    return int(_lib.hpc_step_record_bytes(num_ctas, record_items))


def read_record(record: torch.Tensor, num_ctas: int, record_items: int):
    """The per-CTA records of a single-launch step: (headers RECORD_DTYPE [G], items list of
    ITEM_DTYPE arrays, the first min(n_items, record_items) of each CTA)."""
    raw = record.cpu().numpy()
    stride = RECORD_DTYPE.itemsize + record_items * ITEM_DTYPE.itemsize
    heads = np.empty(num_ctas, dtype=RECORD_DTYPE)
    items = []
    for g in range(num_ctas):
        blk = raw[g * stride:(g + 1) * stride]
        heads[g] = blk[:RECORD_DTYPE.itemsize].view(RECORD_DTYPE)[0]
        n = min(int(heads[g]["n_items"]), record_items)
        items.append(blk[RECORD_DTYPE.itemsize:RECORD_DTYPE.itemsize + n * ITEM_DTYPE.itemsize].view(ITEM_DTYPE))
    return heads, items


def attention(q, k_pages, v_pages, block_table, seq_lens, p: Plan, *, kv_dtype="bf16", kv_layout="HND",
              k_scale=None, v_scale=None, sm_scale=None, out=None, out_dtype=torch.float32, partial_o=None,
              partial_ml=None, status=None, e4m3_kernel="mma", trace=None):
    """Persistent split-KV attention (``hpc_decode_attention``). Returns (out, partial_o, partial_ml)."""
    _need(q, "q", torch.bfloat16)
    dev = q.device
    B, Hq, D = q.shape
    code, num_pages, Hkv, P, lay = _cache(k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, D, dev)
    _tables(block_table, seq_lens, B, dev)
    out = _output(out, (B, Hq, D), out_dtype, dev)
    if partial_o is None or partial_ml is None:
        partial_o, partial_ml = partial_buffers(p, Hq, D, dev)
    status = new_status(dev) if status is None else status
    scale = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    opt = options(e4m3_kernel=e4m3_kernel, trace=trace, device=dev, num_ctas=p.num_ctas)
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_attention(
            _ptr(q), _ptr(k_pages), _ptr(v_pages), code, lay, _ptr(k_scale), _ptr(v_scale), num_pages, P, Hq, Hkv, D,
            _ptr(block_table), block_table.shape[1], _ptr(seq_lens), ctypes.byref(p.raw), scale, _ptr(partial_o),
            _ptr(partial_ml), _ptr(out), _out_code(out), _opt_ref(opt), _ptr(status), _stream(dev)),
            "hpc_decode_attention")
    return out, partial_o, partial_ml


def merge(p: Plan, partial_o, partial_ml, out, num_heads: int, status=None):
    """Log-sum-exp merge of split (request, kv head) pairs (``hpc_merge_states``)."""
    dev = out.device
    _need(partial_o, "partial_o", torch.float32, dev)
    _need(partial_ml, "partial_ml", torch.float32, dev)
    _need(out, "out", (torch.float32, torch.bfloat16), dev)
    status = new_status(dev) if status is None else status
    D = out.shape[-1]
    with torch.cuda.device(dev):
        _check(_lib.hpc_merge_states(_ptr(partial_o), _ptr(partial_ml), ctypes.byref(p.raw), num_heads, D, _ptr(out),
                                     HPC_BF16 if out.dtype == torch.bfloat16 else HPC_FP32, _ptr(status),
                                     _stream(dev)), "hpc_merge_states")
    return out


def prologue(qkv, q_norm_w, k_norm_w, k_pages, v_pages, block_table, seq_lens, num_heads, kv_heads, *,
             kv_dtype="bf16", kv_layout="HND", k_scale=None, v_scale=None, eps=1e-6, rope_theta=1e6, q_out=None,
             status=None):
    """Fused RMSNorm + RoPE + KV-page write of the new token (``hpc_decode_prologue``). Returns q_out."""
    _need(qkv, "qkv", torch.bfloat16)
    dev = qkv.device
    _need(q_norm_w, "q_norm_w", torch.float32, dev)
    _need(k_norm_w, "k_norm_w", torch.float32, dev)
    B, H, D = qkv.shape
    if H != num_heads + 2 * kv_heads:
        raise HpcError("qkv must hold num_heads + 2*kv_heads heads")
    if q_norm_w.numel() != D or k_norm_w.numel() != D:
        raise HpcError("norm weights must hold head_dim values")
    code, num_pages, Hkv, P, lay = _cache(k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, D, dev)
    if Hkv != kv_heads:
        raise HpcError(f"cache has {Hkv} kv heads, expected {kv_heads}")
    _tables(block_table, seq_lens, B, dev)
    if q_out is None:
        q_out = torch.empty((B, num_heads, D), dtype=torch.bfloat16, device=dev)
    _need(q_out, "q_out", torch.bfloat16, dev)
    if tuple(q_out.shape) != (B, num_heads, D):
        raise HpcError("q_out must be [batch, num_heads, head_dim]")
    status = new_status(dev) if status is None else status
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_prologue(
            _ptr(qkv), _ptr(q_norm_w), _ptr(k_norm_w), float(eps), float(rope_theta), _ptr(q_out), _ptr(k_pages),
            _ptr(v_pages), code, lay, _ptr(k_scale), _ptr(v_scale), num_pages, P, _ptr(block_table),
            block_table.shape[1], _ptr(seq_lens), B, num_heads, kv_heads, D, _ptr(status), _stream(dev)),
            "hpc_decode_prologue")
    return q_out


def step_workspace(batch, num_heads, kv_heads, head_dim, num_ctas, device):
    """Zeroed workspace for ``decode_step_fused`` (its merge tickets must start at zero)."""
    n = _lib.hpc_decode_step_workspace_bytes(batch, num_heads, kv_heads, head_dim, num_ctas)
    if n == 0:
        raise HpcError("bad shape for hpc_decode_step_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _grid(num_ctas, dev):
    return torch.cuda.get_device_properties(dev).multi_processor_count if num_ctas is None else int(num_ctas)


def _workspace(ws, nbytes, dev):
    if ws is None:
        return torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    _need(ws, "workspace", torch.uint8, dev)
    return ws


def decode_step_fused(q, k_pages, v_pages, block_table, seq_lens, num_heads, kv_heads, tile_len, *,
                      kv_dtype="bf16", kv_layout="HND", k_scale=None, v_scale=None, num_ctas=None, sm_scale=None,
                      out=None, out_dtype=torch.float32, status=None, workspace=None, item_cost=None,
                      e4m3_kernel="mma", record=None, record_items=0, trace=None, seq_lens_ready=False):
    """One decode step in a single launch (``hpc_decode_step``): in-kernel planning, attention
    and ticket merge. Returns (out, status, workspace); pass the workspace back on later calls.
    item_cost, e4m3_kernel, record / record_items, trace and seq_lens_ready are the call's
    options."""
    _need(q, "q", torch.bfloat16)
    dev = q.device
    B, Hq, D = q.shape
    if Hq != num_heads:
        raise HpcError(f"q has {Hq} heads, expected {num_heads}")
    code, num_pages, Hkv, P, lay = _cache(k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, D, dev)
    if Hkv != kv_heads:
        raise HpcError(f"cache has {Hkv} kv heads, expected {kv_heads}")
    _tables(block_table, seq_lens, B, dev)
    G = _grid(num_ctas, dev)
    out = _output(out, (B, Hq, D), out_dtype, dev)
    status = new_status(dev) if status is None else status
    workspace = _workspace(workspace, _lib.hpc_decode_step_workspace_bytes(B, Hq, Hkv, D, G), dev)
    scale = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    opt = options(item_cost, e4m3_kernel, record, record_items, trace, dev, G, seq_lens_ready=seq_lens_ready)
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_step(
            _ptr(q), _ptr(k_pages), _ptr(v_pages), code, lay, _ptr(k_scale), _ptr(v_scale), num_pages, P, Hq, Hkv, D,
            _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B, tile_len, G, scale, _ptr(workspace),
            workspace.numel(), _ptr(out), _out_code(out), _opt_ref(opt), _ptr(status), _stream(dev)),
            "hpc_decode_step")
    return out, status, workspace


def decode_step_prologue(qkv, q_norm_w, k_norm_w, k_pages, v_pages, block_table, seq_lens, num_heads, kv_heads,
                         tile_len, *, kv_dtype="bf16", kv_layout="HND", k_scale=None, v_scale=None, eps=1e-6,
                         rope_theta=1e6, num_ctas=None, sm_scale=None, out=None, out_dtype=torch.float32,
                         status=None, workspace=None, item_cost=None, record=None, record_items=0, trace=None,
                         seq_lens_ready=False):
    """One decode step in a single launch with the prologue folded in
    (``hpc_decode_step_prologue``): the new token's K/V go into the cache and q is formed from
    qkv inside the attention kernel. Returns (out, status, workspace)."""
    _need(qkv, "qkv", torch.bfloat16)
    dev = qkv.device
    _need(q_norm_w, "q_norm_w", torch.float32, dev)
    _need(k_norm_w, "k_norm_w", torch.float32, dev)
    B, H, D = qkv.shape
    if H != num_heads + 2 * kv_heads:
        raise HpcError("qkv must hold num_heads + 2*kv_heads heads")
    if q_norm_w.numel() != D or k_norm_w.numel() != D:
        raise HpcError("norm weights must hold head_dim values")
    code, num_pages, Hkv, P, lay = _cache(k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, D, dev)
    if Hkv != kv_heads:
        raise HpcError(f"cache has {Hkv} kv heads, expected {kv_heads}")
    _tables(block_table, seq_lens, B, dev)
    G = _grid(num_ctas, dev)
    out = _output(out, (B, num_heads, D), out_dtype, dev)
    status = new_status(dev) if status is None else status
    workspace = _workspace(workspace, _lib.hpc_decode_step_workspace_bytes(B, num_heads, Hkv, D, G), dev)
    scale = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    opt = options(item_cost, "mma", record, record_items, trace, dev, G, seq_lens_ready=seq_lens_ready)
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_step_prologue(
            _ptr(qkv), _ptr(q_norm_w), _ptr(k_norm_w), float(eps), float(rope_theta), _ptr(k_pages), _ptr(v_pages),
            code, lay, _ptr(k_scale), _ptr(v_scale), num_pages, P, num_heads, Hkv, D, _ptr(block_table),
            block_table.shape[1], _ptr(seq_lens), B, tile_len, G, scale, _ptr(workspace), workspace.numel(),
            _ptr(out), _out_code(out), _opt_ref(opt), _ptr(status), _stream(dev)), "hpc_decode_step_prologue")
    return out, status, workspace


def multi_workspace(batch, q_len, num_heads, kv_heads, head_dim, num_ctas, device):
    """Zeroed workspace for ``decode_step_multi``."""
    n = _lib.hpc_decode_step_multi_workspace_bytes(batch, q_len, num_heads, kv_heads, head_dim, num_ctas)
    if n == 0:
        raise HpcError("bad shape for hpc_decode_step_multi_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_step_multi(q, k_pages, v_pages, block_table, seq_lens, kv_heads, tile_len, *, kv_dtype="bf16",
                      kv_layout="HND", k_scale=None, v_scale=None, num_ctas=None, sm_scale=None, out=None,
                      out_dtype=torch.float32, status=None, workspace=None, item_cost=None, record=None,
                      record_items=0, trace=None, multi_kernel="default", seq_lens_ready=False):
    """q_len new tokens per request in one launch (``hpc_decode_step_multi``): q is
    [B, q_len, Hq, D]; query token t of request r sits at position L_r - q_len + t and
    attends causally. multi_kernel: "default", "mma" or "tcgen05". Returns (out [B, q_len, Hq, D],
    status, workspace)."""
    _need(q, "q", torch.bfloat16)
    dev = q.device
    B, T, Hq, D = q.shape
    code, num_pages, Hkv, P, lay = _cache(k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, D, dev)
    if Hkv != kv_heads:
        raise HpcError(f"cache has {Hkv} kv heads, expected {kv_heads}")
    _tables(block_table, seq_lens, B, dev)
    G = _grid(num_ctas, dev)
    out = _output(out, (B, T, Hq, D), out_dtype, dev)
    status = new_status(dev) if status is None else status
    workspace = _workspace(workspace, _lib.hpc_decode_step_multi_workspace_bytes(B, T, Hq, Hkv, D, G), dev)
    scale = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    opt = options(item_cost, "mma", record, record_items, trace, dev, G, multi_kernel, seq_lens_ready)
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_step_multi(
            _ptr(q), T, _ptr(k_pages), _ptr(v_pages), code, lay, _ptr(k_scale), _ptr(v_scale), num_pages, P, Hq, Hkv,
            D, _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B, tile_len, G, scale, _ptr(workspace),
            workspace.numel(), _ptr(out), _out_code(out), _opt_ref(opt), _ptr(status), _stream(dev)),
            "hpc_decode_step_multi")
    return out, status, workspace


def decode_step_lse(q, k_pages, v_pages, block_table, seq_lens, num_heads, kv_heads, tile_len, *, kv_dtype="bf16",
                    kv_layout="HND", k_scale=None, v_scale=None, num_ctas=None, sm_scale=None, out=None, lse=None,
                    status=None, workspace=None, item_cost=None, e4m3_kernel="mma", seq_lens_ready=False):
    """``hpc_decode_step_lse``: the single-launch step, plus the natural-log log-sum-exp of
    every output row. Returns (out fp32 [B, Hq, D], lse fp32 [B, Hq], status, workspace)."""
    _need(q, "q", torch.bfloat16)
    dev = q.device
    B, Hq, D = q.shape
    if Hq != num_heads:
        raise HpcError(f"q has {Hq} heads, expected {num_heads}")
    code, num_pages, Hkv, P, lay = _cache(k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, D, dev)
    if Hkv != kv_heads:
        raise HpcError(f"cache has {Hkv} kv heads, expected {kv_heads}")
    _tables(block_table, seq_lens, B, dev)
    G = _grid(num_ctas, dev)
    out = _output(out, (B, Hq, D), torch.float32, dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev) if lse is None else lse
    _need(lse, "lse", torch.float32, dev)
    if tuple(lse.shape) != (B, Hq):
        raise HpcError("lse must be [batch, num_heads]")
    status = new_status(dev) if status is None else status
    workspace = _workspace(workspace, _lib.hpc_decode_step_workspace_bytes(B, Hq, Hkv, D, G), dev)
    scale = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    opt = options(item_cost, e4m3_kernel, device=dev, seq_lens_ready=seq_lens_ready)
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_step_lse(
            _ptr(q), _ptr(k_pages), _ptr(v_pages), code, lay, _ptr(k_scale), _ptr(v_scale), num_pages, P, Hq, Hkv, D,
            _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B, tile_len, G, scale, _ptr(workspace),
            workspace.numel(), _ptr(out), _out_code(out), _ptr(lse), _opt_ref(opt), _ptr(status), _stream(dev)),
            "hpc_decode_step_lse")
    return out, lse, status, workspace


def merge_lse(outs, lses, out=None, lse_out=None):
    """``hpc_merge_lse``: outs fp32 [parts, rows..., D], lses fp32 [parts, rows...] -> (out, lse)."""
    _need(outs, "outs", torch.float32)
    dev = outs.device
    _need(lses, "lses", torch.float32, dev)
    parts, D = outs.shape[0], outs.shape[-1]
    rows = lses[0].numel()
    if outs[0].numel() != rows * D:
        raise HpcError("outs and lses disagree on the rows")
    out = torch.empty(outs.shape[1:], dtype=torch.float32, device=dev) if out is None else out
    lse_out = torch.empty(lses.shape[1:], dtype=torch.float32, device=dev) if lse_out is None else lse_out
    with torch.cuda.device(dev):
        _check(_lib.hpc_merge_lse(_ptr(outs), _ptr(lses), parts, rows, D, _ptr(out), _ptr(lse_out), _stream(dev)),
               "hpc_merge_lse")
    return out, lse_out


def merge_lse_gather(outs, lses, part_index, out=None, lse_out=None, status=None):
    """``hpc_merge_lse_gather``: outs fp32 [part_rows, Hq, D], lses fp32 [part_rows, Hq], part_index
    int32 [B, max_parts] (-1 unused) -> (out [B, Hq, D], lse [B, Hq])."""
    _need(outs, "outs", torch.float32)
    dev = outs.device
    _need(lses, "lses", torch.float32, dev)
    _need(part_index, "part_index", torch.int32, dev)
    rows, Hq, D = outs.shape
    if tuple(lses.shape) != (rows, Hq) or part_index.dim() != 2:
        raise HpcError("outs [rows, Hq, D], lses [rows, Hq] and part_index [B, max_parts] disagree")
    Bn, mp = part_index.shape
    out = torch.empty((Bn, Hq, D), dtype=torch.float32, device=dev) if out is None else out
    lse_out = torch.empty((Bn, Hq), dtype=torch.float32, device=dev) if lse_out is None else lse_out
    _need(out, "out", torch.float32, dev)
    _need(lse_out, "lse_out", torch.float32, dev)
    with torch.cuda.device(dev):
        _check(_lib.hpc_merge_lse_gather(_ptr(outs), _ptr(lses), rows, _ptr(part_index), mp, Bn, Hq, D, _ptr(out),
                                         _ptr(lse_out), _ptr(status), _stream(dev)), "hpc_merge_lse_gather")
    return out, lse_out


def gather_rows(src, index, out=None, status=None):
    """``hpc_gather_rows``: out[j] = src[index[j]] along the first dimension (rows a multiple of 16 bytes)."""
    _need(src, "src")
    dev = src.device
    _need(index, "index", torch.int32, dev)
    n = index.numel()
    out = torch.empty((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=dev) if out is None else out
    _need(out, "out", src.dtype, dev)
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else out[0].numel() * out.element_size()
    with torch.cuda.device(dev):
        _check(_lib.hpc_gather_rows(_ptr(src), src.shape[0], row_bytes, _ptr(index), n, _ptr(out), _ptr(status),
                                    _stream(dev)), "hpc_gather_rows")
    return out


def gather_pages(block_table, req, col0, width=None, out=None, status=None):
    """``hpc_gather_pages``: out[i][j] = block_table[req[i]][col0[i] + j] (-1 past the table), the
    block-table view of a request-sharded rank's parts. Returns out int32 [n, width]."""
    _need(block_table, "block_table", torch.int32)
    dev = block_table.device
    _need(req, "req", torch.int32, dev)
    _need(col0, "col0", torch.int32, dev)
    if block_table.dim() != 2 or req.numel() != col0.numel():
        raise HpcError("block_table must be 2-D and req / col0 of equal length")
    n = req.numel()
    width = block_table.shape[1] if width is None else int(width)
    out = torch.empty((n, width), dtype=torch.int32, device=dev) if out is None else out
    _need(out, "out", torch.int32, dev)
    if tuple(out.shape) != (n, width):
        raise HpcError("out must be [n, width]")
    with torch.cuda.device(dev):
        _check(_lib.hpc_gather_pages(_ptr(block_table), block_table.shape[0], block_table.shape[1], _ptr(req),
                                     _ptr(col0), n, width, _ptr(out), _ptr(status), _stream(dev)), "hpc_gather_pages")
    return out


def wait_selftest(limit_ns: int, arrive: bool, device, status=None):
    """``hpc_wait_selftest``: the library's bounded wait on a barrier phase that completes at once
    (arrive) or never (not arrive). Returns (status word, waited ns), both device tensors."""
    dev = torch.device(device)
    status = new_status(dev) if status is None else status
    waited = torch.zeros(1, dtype=torch.int64, device=dev)
    with torch.cuda.device(dev):
        _check(_lib.hpc_wait_selftest(int(limit_ns), 1 if arrive else 0, _ptr(status), _ptr(waited), _stream(dev)),
               "hpc_wait_selftest")
    return status, waited


def decode_step(q, k_pages, v_pages, block_table, seq_lens, num_heads, kv_heads, tile_len, *, kv_dtype="bf16",
                kv_layout="HND", k_scale=None, v_scale=None, num_ctas=None, out=None, out_dtype=torch.float32,
                status=None, static_splits=None, e4m3_kernel="mma"):
    """plan -> attention -> merge (three launches) for one decode step; returns (out, plan, status)."""
    dev = q.device
    status = new_status(dev) if status is None else status
    max_seq = block_table.shape[1] * _geometry(k_pages, kv_layout)[2]
    if static_splits:
        p = plan_static(seq_lens, num_heads, kv_heads, tile_len, static_splits, max_seq, status)
    else:
        p = plan(seq_lens, num_heads, kv_heads, tile_len, num_ctas, max_seq, status)
    out, po, pml = attention(q, k_pages, v_pages, block_table, seq_lens, p, kv_dtype=kv_dtype, kv_layout=kv_layout,
                             k_scale=k_scale, v_scale=v_scale, out=out, out_dtype=out_dtype, status=status,
                             e4m3_kernel=e4m3_kernel)
    merge(p, po, pml, out, num_heads, status)
    return out, p, status


NOALLOC_SCRATCH_BYTES = 16 << 20


def decode_step_noalloc(q, k_pages, v_pages, block_table, seq_lens, num_heads, kv_heads, tile_len, *,
                        kv_dtype="bf16", k_scale=None, v_scale=None, num_ctas=None, sm_scale=None, out=None,
                        out_dtype=torch.float32, status=None):
    """One decode step through ``hpc_decode_step_noalloc``: the library keeps the plan and
    partial states in its own static device array, for callers that cannot allocate device
    memory. Returns (out, status). Calls that overlap on the GPU share that array; keep
    them on one stream. The cache is HND."""
    _need(q, "q", torch.bfloat16)
    dev = q.device
    B, Hq, D = q.shape
    if Hq != num_heads:
        raise HpcError(f"q has {Hq} heads, expected {num_heads}")
    code, num_pages, Hkv, P, _ = _cache(k_pages, v_pages, kv_dtype, "HND", k_scale, v_scale, D, dev)
    if Hkv != kv_heads:
        raise HpcError(f"cache has {Hkv} kv heads, expected {kv_heads}")
    _tables(block_table, seq_lens, B, dev)
    G = _grid(num_ctas, dev)
    out = _output(out, (B, Hq, D), out_dtype, dev)
    status = new_status(dev) if status is None else status
    _need(status, "status", torch.int32, dev)
    scale = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    with torch.cuda.device(dev):
        _check(_lib.hpc_decode_step_noalloc(
            _ptr(q), _ptr(k_pages), _ptr(v_pages), code, _ptr(k_scale), _ptr(v_scale), num_pages, P, Hq, Hkv, D,
            _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B, tile_len, G, scale, _ptr(out),
            _out_code(out), _ptr(status), _stream(dev)), "hpc_decode_step_noalloc")
    return out, status


def launch_info(head_dim, kv_dtype, page_size, tile_len, ctas_per_sm=1, e4m3_kernel="mma"):
    st, sm, th = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.hpc_attention_launch_info(head_dim, _KV_DTYPES[kv_dtype], page_size, tile_len, ctas_per_sm,
                                          E4M3_KERNELS[e4m3_kernel], ctypes.byref(st), ctypes.byref(sm),
                                          ctypes.byref(th)), "hpc_attention_launch_info")
    return {"stages": st.value, "smem_bytes": sm.value, "threads": th.value}
