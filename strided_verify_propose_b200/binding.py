"""ctypes binding of libisd.so (argument marshalling only).

Every step of the ISD path runs in the library's CUDA kernels; this module
only loads the library, mirrors the C structs of ``include/isd.h``, lays
weights out in the ABI's layout and passes device pointers and the current
CUDA stream. It never falls back to a CPU or PyTorch implementation: if the
library is missing the first call raises.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libisd.so")

ISD_OK = 0
ISD_E_INVALID, ISD_E_UNSUPPORTED = -1, -2
ISD_DEV_POOL_EXHAUSTED = 0x01
ISD_DEV_TABLE_FULL = 0x02
ISD_DEV_BAD_TOKEN = 0x04
ISD_DEV_BAD_PAGE = 0x08
ISD_DEV_TIMEOUT = 0x10
ISD_DEV_BAD_STATE = 0x20

PROPOSE_ARGMAX, PROPOSE_SAMPLE = 0x0, 0x1
VERIFY_SAMPLE, VERIFY_GREEDY = 0x0, 0x2
USE_LORA = 0x4

EXPORTS = ("isd_init", "isd_load_gated_lora", "isd_step", "isd_prefill", "isd_last_launch_count",
           "isd_last_error", "isd_destroy", "isd_gemm_bf16", "isd_attention_workspace_bytes",
           "isd_paged_attention", "isd_accept_workspace_bytes", "isd_accept_propose",
           "isd_profile_enable", "isd_profile_read", "isd_profile_class_name",
           "isd_accept_propose_noalloc", "isd_gemm_workspace_bytes", "isd_gemm_bf16_single",
           "isd_gemm_plan", "isd_attention_split", "isd_set_wait_limit")
PROF_CLASSES = 16


class ModelCfg(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("hidden", C.c_int32), ("n_q_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("intermediate", C.c_int32),
                ("vocab", C.c_int32), ("rope_theta", C.c_float), ("rms_eps", C.c_float),
                ("mask_token_id", C.c_int32), ("page_size", C.c_int32), ("max_batch", C.c_int32),
                ("max_rows", C.c_int32), ("max_position", C.c_int32)]


_PP = C.POINTER(C.c_void_p)


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("lm_head", C.c_void_p), ("final_norm", C.c_void_p),
                ("w_qkv", _PP), ("w_o", _PP), ("w_gate_up", _PP), ("w_down", _PP),
                ("attn_norm", _PP), ("mlp_norm", _PP), ("q_norm", _PP), ("k_norm", _PP)]


class Lora(C.Structure):
    _fields_ = [("rank", C.c_int32), ("scale", C.c_float), ("A", _PP * 7), ("B", _PP * 7)]


class Batch(C.Structure):
    _fields_ = [("batch", C.c_int32), ("stride_n", C.c_int32), ("flags", C.c_int32),
                ("seq_len", C.c_void_p), ("n_draft", C.c_void_p), ("logits_out", C.c_void_p)]


class KV(C.Structure):
    _fields_ = [("k_pool", C.c_void_p), ("v_pool", C.c_void_p), ("page_table", C.c_void_p),
                ("free_list", C.c_void_p), ("free_head", C.c_void_p), ("num_pages", C.c_int32),
                ("max_pages_per_req", C.c_int32), ("free_count", C.c_int32)]


_lib = None


def lib():
    """Load libisd.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m strided_verify_propose_b200.build`")
    L = C.CDLL(LIB_PATH)
    vp, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
    L.isd_init.argtypes = [C.POINTER(ModelCfg), C.POINTER(Weights), C.POINTER(vp)]
    L.isd_load_gated_lora.argtypes = [vp, C.POINTER(Lora)]
    L.isd_step.argtypes = [vp, C.POINTER(Batch), C.POINTER(KV), vp, vp, vp, vp, vp, vp, vp]
    L.isd_prefill.argtypes = [vp, C.POINTER(KV), vp, i32, C.POINTER(i32), i32, i32, vp, vp, vp,
                              vp, vp]
    L.isd_last_launch_count.argtypes = [vp]
    L.isd_last_error.restype = C.c_char_p
    L.isd_destroy.argtypes = [vp]
    L.isd_destroy.restype = None
    L.isd_gemm_bf16.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp]
    L.isd_gemm_workspace_bytes.argtypes = [i32, i32, i32]
    L.isd_gemm_workspace_bytes.restype = sz
    L.isd_gemm_bf16_single.argtypes = [vp, vp, vp, i32, i32, i32, vp, sz, vp, vp]
    L.isd_gemm_plan.argtypes = [i32, i32, i32, i32, i32, i32, C.POINTER(i32)]
    L.isd_attention_split.argtypes = [i32] * 7 + [C.POINTER(i32), i32, C.POINTER(i32), i32,
                                                  C.POINTER(i32), C.POINTER(i32)]
    L.isd_attention_workspace_bytes.argtypes = [i32] * 7
    L.isd_attention_workspace_bytes.restype = sz
    L.isd_paged_attention.argtypes = [vp, vp, vp, vp, vp] + [i32] * 10 + [vp, vp, sz, vp, vp]
    L.isd_accept_workspace_bytes.argtypes = [i32, i32, i32]
    L.isd_accept_workspace_bytes.restype = sz
    L.isd_accept_propose.argtypes = [vp, C.POINTER(Batch), C.POINTER(KV), i32, i32, vp, vp, vp,
                                     vp, vp, vp, sz, vp, vp]
    L.isd_accept_propose_noalloc.argtypes = [vp, C.POINTER(Batch), C.POINTER(KV), i32, i32, vp,
                                             vp, vp, vp, vp, vp, vp]
    L.isd_set_wait_limit.argtypes = [C.c_longlong]
    L.isd_profile_enable.argtypes = [vp, C.c_int]
    L.isd_profile_read.argtypes = [vp, C.POINTER(C.c_double), C.POINTER(i32)]
    L.isd_profile_class_name.argtypes = [C.c_int]
    L.isd_profile_class_name.restype = C.c_char_p
    _lib = L
    return L


def check(rc: int) -> None:
    if rc != ISD_OK:
        raise RuntimeError(f"libisd error {rc}: {lib().isd_last_error().decode()}")


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream():
    import torch
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr_array(ts: Sequence) -> C.Array:
    arr = (C.c_void_p * len(ts))(*[int(t.data_ptr()) for t in ts])
    return arr


# --------------------------------------------------------------- weights ---

def pack_weights(shape, w: Dict[str, object], device="cuda") -> Dict[str, object]:
    """Device tensors in the ABI layout from per-matrix weights (numpy or torch):
    fused QKV rows [q | k | v], gate/up interleaved in blocks of 16 rows."""
    import torch

    def bf(a):
        t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))
        return t.to(device=device, dtype=torch.bfloat16).contiguous()

    def f32(a):
        t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))
        return t.to(device=device, dtype=torch.float32).contiguous()

    out = {"embed": bf(w["embed"]), "lm_head": bf(w["lm_head"]), "final_norm": f32(w["final_norm"]),
           "layers": []}
    I = shape.intermediate
    for lw in w["layers"]:
        qkv = torch.cat([bf(lw["wq"]), bf(lw["wk"]), bf(lw["wv"])], 0).contiguous()
        g = bf(lw["w_gate"]).view(I // 16, 16, shape.hidden)
        u = bf(lw["w_up"]).view(I // 16, 16, shape.hidden)
        gu = torch.stack([g, u], 1).reshape(2 * I, shape.hidden).contiguous()
        out["layers"].append({"w_qkv": qkv, "w_o": bf(lw["wo"]), "w_gate_up": gu,
                              "w_down": bf(lw["w_down"]), "attn_norm": f32(lw["attn_norm"]),
                              "mlp_norm": f32(lw["mlp_norm"]), "q_norm": f32(lw["q_norm"]),
                              "k_norm": f32(lw["k_norm"])})
    return out


def random_device_weights(shape, seed: int = 0, std: float = 0.02, device="cuda"):
    """Random-init weights generated directly on the device in the ABI layout
    (for throughput runs at full size; the oracle never sees these)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    def rnd(*s):
        t = torch.empty(*s, device=device, dtype=torch.bfloat16)
        t.normal_(0.0, std, generator=gen)
        return t

    h, I = shape.hidden, shape.intermediate
    ones = lambda n: torch.ones(n, device=device, dtype=torch.float32)
    out = {"embed": rnd(shape.vocab, h), "lm_head": rnd(shape.vocab, h), "final_norm": ones(h),
           "layers": []}
    for _ in range(shape.n_layers):
        out["layers"].append({"w_qkv": rnd(shape.qkv_dim, h), "w_o": rnd(h, shape.q_dim),
                              "w_gate_up": rnd(2 * I, h), "w_down": rnd(h, I),
                              "attn_norm": ones(h), "mlp_norm": ones(h),
                              "q_norm": ones(shape.head_dim), "k_norm": ones(shape.head_dim)})
    return out


def random_device_lora(shape, rank: int = 128, seed: int = 0, std: float = 0.01, device="cuda"):
    """Random gated-LoRA adapters on the device, per layer {target: (A [in, r], B [r, out])}
    (for throughput runs; the oracle never sees these)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 7919)
    h, i = shape.hidden, shape.intermediate
    dims = {"q": (h, shape.q_dim), "k": (h, shape.kv_dim), "v": (h, shape.kv_dim),
            "o": (shape.q_dim, h), "gate": (h, i), "up": (h, i), "down": (i, h)}

    def rnd(*s):
        t = torch.empty(*s, device=device, dtype=torch.bfloat16)
        t.normal_(0.0, std, generator=gen)
        return t
    return [{t: (rnd(dims[t][0], rank), rnd(rank, dims[t][1])) for t in dims}
            for _ in range(shape.n_layers)]


class Model:
    """An isd_ctx over device weights in the ABI layout (see pack_weights)."""

    def __init__(self, shape, dev_weights, max_batch: int, max_rows: int, max_position: int):
        self.shape = shape
        self.w = dev_weights
        L = lib()
        cfg = ModelCfg(shape.n_layers, shape.hidden, shape.n_q_heads, shape.n_kv_heads,
                       shape.head_dim, shape.intermediate, shape.vocab, shape.rope_theta,
                       shape.rms_eps, shape.mask_token_id, shape.page_size, max_batch, max_rows,
                       max_position)
        layers = dev_weights["layers"]
        self._arrays = {k: _ptr_array([lw[k] for lw in layers]) for k in
                        ("w_qkv", "w_o", "w_gate_up", "w_down", "attn_norm", "mlp_norm",
                         "q_norm", "k_norm")}
        cast = lambda a: C.cast(a, _PP)
        w = Weights(_ptr(dev_weights["embed"]), _ptr(dev_weights["lm_head"]),
                    _ptr(dev_weights["final_norm"]),
                    *[cast(self._arrays[k]) for k in ("w_qkv", "w_o", "w_gate_up", "w_down",
                                                      "attn_norm", "mlp_norm", "q_norm", "k_norm")])
        h = C.c_void_p()
        check(L.isd_init(C.byref(cfg), C.byref(w), C.byref(h)))
        self.ctx = h
        self.max_batch, self.max_rows, self.max_position = max_batch, max_rows, max_position

    def close(self):
        if self.ctx:
            lib().isd_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def launches(self) -> int:
        return int(lib().isd_last_launch_count(self.ctx))

    def load_lora(self, lora_layers, rank: int = 128, scale: float = 1.0, device="cuda"):
        """Attach a gated LoRA. lora_layers: per layer {target: (A [in, r], B [r, out])}
        (numpy or torch, as synth.lora_weights returns them); passed to the library
        as the nn.Linear weights A^T [r][in] and B^T [out][r] in bf16."""
        import torch
        targets = ("q", "k", "v", "o", "gate", "up", "down")

        def bf(a):
            t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))
            return t.to(device=device, dtype=torch.bfloat16).t().contiguous()

        self._lora = [{t: (bf(ll[t][0]), bf(ll[t][1])) for t in targets} for ll in lora_layers]
        self._lora_arrays = []
        lo = Lora()
        lo.rank = rank
        lo.scale = scale
        for i, t in enumerate(targets):
            a = _ptr_array([ll[t][0] for ll in self._lora])
            b = _ptr_array([ll[t][1] for ll in self._lora])
            self._lora_arrays += [a, b]
            lo.A[i] = C.cast(a, _PP)
            lo.B[i] = C.cast(b, _PP)
        check(lib().isd_load_gated_lora(self.ctx, C.byref(lo)))

    def profile(self, enable: bool) -> None:
        check(lib().isd_profile_enable(self.ctx, 1 if enable else 0))

    def profile_read(self) -> Dict[str, tuple]:
        """{kernel class: (total ms, launches)} since the last read (synchronises)."""
        ms = (C.c_double * PROF_CLASSES)()
        cnt = (C.c_int32 * PROF_CLASSES)()
        check(lib().isd_profile_read(self.ctx, ms, cnt))
        out = {}
        for i in range(PROF_CLASSES):
            if cnt[i]:
                out[lib().isd_profile_class_name(i).decode()] = (float(ms[i]), int(cnt[i]))
        return out


# ------------------------------------------------------------- KV / state ---

class KVCache:
    """Zero-initialised paged KV pools, page table and free list on the device."""

    def __init__(self, shape, num_pages: int, page_table: np.ndarray, free_list: np.ndarray,
                 device="cuda", n_layers: Optional[int] = None):
        import torch
        L = shape.n_layers if n_layers is None else n_layers
        dims = (max(L, 1), num_pages, shape.n_kv_heads, shape.page_size, shape.head_dim)
        self.k_pool = torch.zeros(dims, device=device, dtype=torch.bfloat16)
        self.v_pool = torch.zeros(dims, device=device, dtype=torch.bfloat16)
        self.page_table = torch.from_numpy(np.ascontiguousarray(page_table, np.int32)).to(device)
        fl = np.ascontiguousarray(free_list, np.int32)
        self.free_list = torch.from_numpy(fl if len(fl) else np.zeros(1, np.int32)).to(device)
        self.free_count = int(len(fl))
        self.free_head = torch.zeros(1, device=device, dtype=torch.int32)
        self.num_pages = num_pages
        self.max_pages_per_req = int(page_table.shape[1])

    def c(self) -> KV:
        return KV(_ptr(self.k_pool), _ptr(self.v_pool), _ptr(self.page_table), _ptr(self.free_list),
                  _ptr(self.free_head), self.num_pages, self.max_pages_per_req, self.free_count)


class StepState:
    """Per-request device state of an ISD run."""

    def __init__(self, batch: int, stride_n: int, vocab: int, sample: bool, device="cuda"):
        import torch
        i32 = dict(device=device, dtype=torch.int32)
        self.B, self.N = batch, stride_n
        self.seq_len = torch.zeros(batch, **i32)
        self.n_draft = torch.zeros(batch, **i32)
        self.pending = torch.zeros(batch, stride_n, **i32)
        self.accepted = torch.zeros(batch, **i32)
        self.committed = torch.zeros(batch, stride_n, **i32)
        self.status = torch.zeros(1, **i32)
        self.q_cache = (torch.zeros(batch, max(stride_n - 1, 1), vocab, device=device,
                                    dtype=torch.float32) if sample else None)


def step(model: Model, kv: KVCache, st: StepState, uniforms, flags: int = 0, logits_out=None):
    """One isd_step on the current stream (uniforms: [B, 2N-1] float32 device)."""
    b = Batch(st.B, st.N, flags, _ptr(st.seq_len), _ptr(st.n_draft), _ptr(logits_out))
    kvc = kv.c()
    check(lib().isd_step(model.ctx, C.byref(b), C.byref(kvc), _ptr(st.pending), _ptr(st.q_cache),
                         _ptr(uniforms), _ptr(st.accepted), _ptr(st.committed), _ptr(st.status),
                         _stream()))


class StepGraph:
    """`steps` consecutive isd_step calls captured once into a CUDA graph.

    The graph holds the launches of every kernel of the steps with their
    arguments fixed: the model, cache and state objects given here, and a
    static uniforms buffer `u` of shape [steps, B, 2N-1] that replay() fills.
    Replaying runs the same device work as calling step() `steps` times with
    those uniforms, without host launch overhead. Run at least one eager step
    first (the library sets kernel attributes on first use) and keep every
    object alive while the graph is used.
    """

    def __init__(self, model: Model, kv: KVCache, st: StepState, steps: int, flags: int = 0):
        import torch
        self.steps = steps
        R = 2 * st.N - 1
        self.u = torch.zeros(steps, st.B, R, device=st.seq_len.device, dtype=torch.float32)
        # per-step acceptance counts, recorded inside the graph
        self.accepted = torch.zeros(steps, st.B, device=st.seq_len.device, dtype=torch.int32)
        self.graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(self.graph, stream=side):
                for i in range(steps):
                    step(model, kv, st, self.u[i], flags)
                    self.accepted[i].copy_(st.accepted)
        torch.cuda.current_stream().wait_stream(side)

    def replay(self, uniforms=None):
        """Run the captured steps (uniforms: [steps, B, 2N-1] float32 device, optional)."""
        if uniforms is not None:
            self.u.copy_(uniforms)
        self.graph.replay()


def prefill(model: Model, kv: KVCache, st: StepState, prompts: List[np.ndarray]):
    """isd_prefill of one prompt per request (host token lists)."""
    import torch
    B = len(prompts)
    max_len = max(len(p) for p in prompts)
    tok = np.zeros((B, max_len), np.int32)
    for b, p in enumerate(prompts):
        tok[b, :len(p)] = p
    tok_d = torch.from_numpy(tok).to(st.seq_len.device)
    lens = (C.c_int32 * B)(*[len(p) for p in prompts])
    check(lib().isd_prefill(model.ctx, C.byref(kv.c()), _ptr(tok_d), max_len, lens, B, st.N,
                            _ptr(st.seq_len), _ptr(st.n_draft), _ptr(st.pending), _ptr(st.status),
                            _stream()))


# ------------------------------------------------------ component calls ---

def set_wait_limit(cycles: int) -> None:
    """Cycle limit of the library's bounded device waits (0: the default)."""
    check(lib().isd_set_wait_limit(int(cycles)))


def gemm_bf16(w, x, split_k: int = 1, status=None):
    """Y[split][m][n] partial sums of X W^T (torch bf16 device tensors)."""
    import torch
    n, k = w.shape
    m = x.shape[0]
    y = torch.empty(split_k, m, n, device=x.device, dtype=torch.float32)
    st = status if status is not None else torch.zeros(1, device=x.device, dtype=torch.int32)
    check(lib().isd_gemm_bf16(_ptr(w), _ptr(x), _ptr(y), m, n, k, split_k, _ptr(st), _stream()))
    return y


GEMM_PLAN_FIELDS = ("n_pad", "n_chunks", "splits", "kb_per_split", "n_mma", "mma_n", "box_rows",
                    "n_boxes", "stages", "pair", "streamk", "units", "tmem_cols", "smem_bytes")


def gemm_plan(m: int, n: int, k: int, single: bool = False, max_splits: int = 8,
              num_sms: int = 148) -> Optional[dict]:
    """The library's tile plan for an m x n x k projection (host only), or None."""
    out = (C.c_int32 * len(GEMM_PLAN_FIELDS))()
    if lib().isd_gemm_plan(m, n, k, int(single), max_splits, num_sms, out) != 0:
        return None
    return dict(zip(GEMM_PLAN_FIELDS, list(out)))


ATTN_SEG_FIELDS = ("cta", "request", "kv_head", "tile0", "tiles", "slot")


def attention_split(batch: int, rows_per_req: int, n_q: int, n_kv: int, head_dim: int,
                    max_pages_per_req: int, page_size: int, kend, num_sms: int = 148):
    """The tcgen05 attention kernel's work split (host only): an int32 array
    [segments][ATTN_SEG_FIELDS] in CTA order and the partial slots per
    (request, KV head); None when that kernel does not serve the shape."""
    import numpy as np
    ke = np.ascontiguousarray(np.asarray(kend, dtype=np.int32))
    if ke.shape != (batch,):
        raise ValueError("kend needs one key count per request")
    kp = ke.ctypes.data_as(C.POINTER(C.c_int32))
    n, mp = C.c_int32(0), C.c_int32(0)
    L = lib()
    rc = L.isd_attention_split(batch, rows_per_req, n_q, n_kv, head_dim, max_pages_per_req,
                               page_size, kp, num_sms, None, 0, C.byref(n), C.byref(mp))
    if rc == ISD_E_UNSUPPORTED:
        return None
    seg = np.zeros((max(n.value, 1), len(ATTN_SEG_FIELDS)), np.int32)
    check(L.isd_attention_split(batch, rows_per_req, n_q, n_kv, head_dim, max_pages_per_req,
                                page_size, kp, num_sms, seg.ctypes.data_as(C.POINTER(C.c_int32)),
                                seg.shape[0], C.byref(n), C.byref(mp)))
    return seg[:n.value], mp.value


def gemm_workspace(m: int, n: int, k: int, device="cuda"):
    """A zeroed workspace for gemm_bf16_single at this shape (None if not needed)."""
    import torch
    nb = int(lib().isd_gemm_workspace_bytes(m, n, k))
    return torch.zeros(nb, device=device, dtype=torch.uint8) if nb else None


def gemm_bf16_single(w, x, workspace=None, status=None):
    """Y[m][n] = X W^T as one fp32 slice (stream-K when the tiles overfill a wave)."""
    import torch
    n, k = w.shape
    m = x.shape[0]
    y = torch.empty(m, n, device=x.device, dtype=torch.float32)
    st = status if status is not None else torch.zeros(1, device=x.device, dtype=torch.int32)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel())
    check(lib().isd_gemm_bf16_single(_ptr(w), _ptr(x), _ptr(y), m, n, k, ws_ptr, ws_bytes, _ptr(st),
                                     _stream()))
    return y


def attention_workspace(batch: int, rows_per_req: int, n_q: int, n_kv: int, head_dim: int,
                        max_pages_per_req: int, page_size: int, device="cuda"):
    """Workspace for isd_paged_attention at these sizes (scratch only: any
    later launch that fits may reuse it)."""
    import torch
    n = int(lib().isd_attention_workspace_bytes(batch, rows_per_req, n_q, n_kv, head_dim,
                                                max_pages_per_req, page_size))
    return torch.empty(n, device=device, dtype=torch.uint8)


def paged_attention(q, row_pos, k_pool, v_pool, page_table, rows_per_req: int, layer: int = 0,
                    status=None, workspace=None):
    """Attention of rows q [B*R, n_q, hd] over the paged pools (torch device
    tensors). workspace: from attention_workspace, else a fresh one."""
    import torch
    n_layers, num_pages, n_kv, page_size, hd = k_pool.shape
    rows, n_q, _ = q.shape
    B = rows // rows_per_req
    maxp = page_table.shape[1]
    ws = workspace if workspace is not None else attention_workspace(
        B, rows_per_req, n_q, n_kv, hd, maxp, page_size, q.device)
    ws_bytes = ws.numel()
    out = torch.empty(rows, n_q * hd, device=q.device, dtype=torch.bfloat16)
    st = status if status is not None else torch.zeros(1, device=q.device, dtype=torch.int32)
    check(lib().isd_paged_attention(_ptr(q), _ptr(row_pos), _ptr(k_pool), _ptr(v_pool),
                                    _ptr(page_table), B, rows_per_req, n_q, n_kv, hd, page_size,
                                    num_pages, maxp, n_layers, layer, _ptr(out), _ptr(ws), ws_bytes,
                                    _ptr(st), _stream()))
    return out


def accept_propose(logits, st: StepState, kv: KVCache, page_size: int, uniforms, flags: int = 0):
    """Verify / resample / propose + bookkeeping from given logits [B*(2N-1), V]."""
    import torch
    V = logits.shape[1]
    ws_bytes = int(lib().isd_accept_workspace_bytes(st.B, st.N, V))
    ws = torch.empty(ws_bytes, device=logits.device, dtype=torch.uint8)
    b = Batch(st.B, st.N, flags, _ptr(st.seq_len), _ptr(st.n_draft), None)
    check(lib().isd_accept_propose(_ptr(logits), C.byref(b), C.byref(kv.c()), page_size, V,
                                   _ptr(st.pending), _ptr(st.q_cache), _ptr(uniforms),
                                   _ptr(st.accepted), _ptr(st.committed), _ptr(ws), ws_bytes,
                                   _ptr(st.status), _stream()))


def accept_propose_noalloc(logits, st: StepState, kv: KVCache, page_size: int, uniforms,
                           flags: int = 0):
    """accept_propose without any device allocation: the library's fixed
    scratch array stands in for the workspace (for callers that cannot
    allocate device memory)."""
    b = Batch(st.B, st.N, flags, _ptr(st.seq_len), _ptr(st.n_draft), None)
    check(lib().isd_accept_propose_noalloc(_ptr(logits), C.byref(b), C.byref(kv.c()), page_size,
                                           logits.shape[1], _ptr(st.pending), _ptr(st.q_cache),
                                           _ptr(uniforms), _ptr(st.accepted), _ptr(st.committed),
                                           _ptr(st.status), _stream()))
