"""Python binding of libet, the event-tensor megakernel library for B200.

Argument marshalling only: every function has the name and meaning of the C
entry point in ``include/et.h``.  Tensor arguments may be torch tensors
(their ``data_ptr()`` is passed), integers (device addresses) or None (NULL).
``stream`` defaults to torch's current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels; importing this package
fails if ``libet.so`` has not been built (``python -m
event_driven_persistent_b200.build``).
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libet.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libet.so is missing: build it with `python event_driven_persistent_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

# ------------------------------------------------------------ constants --
ET_OK, ET_ERR_INVALID, ET_ERR_CUDA, ET_ERR_TIMEOUT, ET_ERR_OOM, ET_ERR_UNSUPPORTED, ET_ERR_PENDING, ET_ERR_INTERNAL = range(8)
ET_SCHED_STATIC, ET_SCHED_DYNAMIC, ET_SCHED_UNFUSED, ET_SCHED_HYBRID = 0, 1, 2, 3
ET_GRAPH_SPLITK, ET_GRAPH_MLP, ET_GRAPH_MOE, ET_GRAPH_DECODE, ET_GRAPH_MOE_MLP = 0, 1, 2, 3, 4
ET_DEBUG_TRACE, ET_DEBUG_DELAY, ET_DEBUG_BAD_COUNT, ET_DEBUG_CTA_TIMES = 1, 2, 4, 8
SCHED = {"static": ET_SCHED_STATIC, "dynamic": ET_SCHED_DYNAMIC, "unfused": ET_SCHED_UNFUSED,
         "hybrid": ET_SCHED_HYBRID}


class EtError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        msg = _lib.et_status_str(status).decode()
        super().__init__("%s: %s (status %d)" % (where, msg, status) if where else msg)


class et_graph_desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "kind", "sched", "max_T", "hidden", "inter", "n_experts", "top_k", "splitk_cols", "splitk_chunk",
        "splitk_tile_rows")] + [("rms_eps", ctypes.c_float)] + [(n, ctypes.c_int) for n in (
            "fetch_batch", "debug_flags", "device", "n_ctas")] + [("timeout_ms", ctypes.c_float)] + [
            (n, ctypes.c_int) for n in ("n_heads", "n_kv_heads", "head_dim", "max_ctx")] + [
            ("rope_base", ctypes.c_float), ("mlp_inter", ctypes.c_int), ("moe_xp_min_T", ctypes.c_int)]


class et_graph_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "kind", "sched", "max_T", "n_ctas", "threads", "smem_bytes", "fetch_batch", "hidden", "inter",
        "n_experts", "top_k", "splitk_cols", "splitk_chunk", "splitk_tile_rows", "mlp_gu_tile", "mlp_down_tile",
        "mlp_kchunk", "moe_tt", "moe_gt", "moe_tkt", "moe_bm", "moe_n1_tile", "moe_n2_tile", "moe_cb",
        "dec_split", "dec_qkv_kc", "dec_o_kc")]


class et_decode_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("g1", "Wqkv", "gq", "gk", "Wo", "g2", "Wgu", "Wd")]


class et_trace_record(ctypes.Structure):
    _fields_ = [("op", ctypes.c_int32), ("a", ctypes.c_int32), ("b", ctypes.c_int32), ("sm", ctypes.c_int32),
                ("start", ctypes.c_uint32), ("end", ctypes.c_uint32), ("t_fetch", ctypes.c_uint64),
                ("t_ready", ctypes.c_uint64), ("t_acc", ctypes.c_uint64), ("t_end", ctypes.c_uint64)]


class et_event_count(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("index", ctypes.c_int32), ("count", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_sigs = {
    "et_build_graph": ([ctypes.POINTER(et_graph_desc), ctypes.POINTER(_P)], _I),
    "et_run_splitk": ([_P, _P, _I, _P, _P, _P], _I),
    "et_run_mlp": ([_P, _I, _P, _P, _P, _P, _P, _P], _I),
    "et_run_moe": ([_P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P], _I),
    "et_run_splitk_noalloc": ([_P, _I, _P, _P, _P], _I),
    "et_run_splitk_two_launch": ([_P, _I, _I, _I, _P, _P, _P], _I),
    "et_run_decode": ([_P, _I, _P, _P, ctypes.POINTER(et_decode_weights), _P, _P, _P, _P, _P], _I),
    "et_run_moe_mlp": ([_P, _I] + [_P] * 11, _I),
    "et_sync_status": ([_P, _P], _I),
    "et_get_trace": ([_P, _P, ctypes.c_size_t, ctypes.POINTER(_I)], _I),
    "et_get_info": ([_P, ctypes.POINTER(et_graph_info)], _I),
    "et_get_diag": ([_P, ctypes.POINTER(ctypes.c_int32)], _I),
    "et_get_event_counts": ([_P, _P, _I, ctypes.POINTER(_I)], _I),
    "et_destroy_graph": ([_P], None),
    "et_status_str": ([_I], ctypes.c_char_p),
}
for _name, (_args, _res) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def _ptr(x):
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    return int(x)


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream
    return int(s)


def _check(status, where):
    if status != ET_OK:
        raise EtError(status, where)


# ------------------------------------------------------------ entry points --
def et_build_graph(kind, sched, max_T, **dims):
    """Build a graph; returns its handle (an int).  `dims` are et_graph_desc fields."""
    d = et_graph_desc()
    d.kind = kind
    d.sched = SCHED[sched] if isinstance(sched, str) else sched
    d.max_T = max_T
    for k, v in dims.items():
        setattr(d, k, v)
    h = _P()
    _check(_lib.et_build_graph(ctypes.byref(d), ctypes.byref(h)), "et_build_graph")
    return h.value


def et_run_splitk(g, A, n_rows, Bpart, C, stream=None):
    _check(_lib.et_run_splitk(g, _ptr(A), n_rows, _ptr(Bpart), _ptr(C), _stream(stream)), "et_run_splitk")


def et_run_splitk_two_launch(A, n_rows, cols, chunk, Bpart, C, stream=None):
    """Control: split-K as two plain kernel launches (partials, finals)."""
    _check(_lib.et_run_splitk_two_launch(_ptr(A), n_rows, cols, chunk, _ptr(Bpart), _ptr(C), _stream(stream)),
           "et_run_splitk_two_launch")


def et_run_splitk_noalloc(A, n_rows, Bpart, C, stream=None):
    """Allocation-free split-K (synchronous); returns the status code."""
    return _lib.et_run_splitk_noalloc(_ptr(A), n_rows, _ptr(Bpart), _ptr(C), _stream(stream))


def et_run_mlp(g, B, X, gamma, Wgu, Wd, Y, stream=None):
    _check(_lib.et_run_mlp(g, B, _ptr(X), _ptr(gamma), _ptr(Wgu), _ptr(Wd), _ptr(Y), _stream(stream)),
           "et_run_mlp")


def et_run_moe(g, T, X, Wr, bias, W1, W2, Y, topk=None, topk_w=None, indptr=None, perm=None, logits=None,
               stream=None):
    _check(_lib.et_run_moe(g, T, _ptr(X), _ptr(Wr), _ptr(bias), _ptr(W1), _ptr(W2), _ptr(Y), _ptr(topk),
                           _ptr(topk_w), _ptr(indptr), _ptr(perm), _ptr(logits), _stream(stream)), "et_run_moe")


def et_run_moe_mlp(g, T, X, Wr, bias, W1, W2, gamma, Wgu, Wd, Y1, Y2, stream=None):
    _check(_lib.et_run_moe_mlp(g, T, _ptr(X), _ptr(Wr), _ptr(bias), _ptr(W1), _ptr(W2), _ptr(gamma), _ptr(Wgu),
                               _ptr(Wd), _ptr(Y1), _ptr(Y2), _stream(stream)), "et_run_moe_mlp")


def et_run_decode(g, B, X, pos, w, Kc, Vc, Y, h1=None, stream=None):
    """w: dict or object with g1, Wqkv, gq, gk, Wo, g2, Wgu, Wd (tensors or addresses)."""
    ws = et_decode_weights()
    for f, _ in et_decode_weights._fields_:
        setattr(ws, f, _ptr(w[f] if isinstance(w, dict) else getattr(w, f)))
    _check(_lib.et_run_decode(g, B, _ptr(X), _ptr(pos), ctypes.byref(ws), _ptr(Kc), _ptr(Vc), _ptr(Y), _ptr(h1),
                              _stream(stream)), "et_run_decode")


def et_sync_status(g, stream=None):
    """Returns the status code (0 = ok); does not raise on device errors."""
    return _lib.et_sync_status(g, _stream(stream))


def et_get_trace(g):
    """List of (op, a, b, sm, start, end, t_fetch, t_ready, t_acc, t_end)
    tuples of the last traced run (tickets, then %globaltimer ns)."""
    n = _I(0)
    _check(_lib.et_get_trace(g, None, 0, ctypes.byref(n)), "et_get_trace")
    buf = (et_trace_record * max(n.value, 1))()
    _check(_lib.et_get_trace(g, ctypes.cast(buf, _P), ctypes.sizeof(buf), ctypes.byref(n)), "et_get_trace")
    return [(r.op, r.a, r.b, r.sm, r.start, r.end, r.t_fetch, r.t_ready, r.t_acc, r.t_end) for r in buf[:n.value]]


def et_get_event_counts(g):
    """List of (kind, index, count): notifications each event of the last
    run received (kind = ET_EV_* code of include/et.h)."""
    n = _I(0)
    _check(_lib.et_get_event_counts(g, None, 0, ctypes.byref(n)), "et_get_event_counts")
    buf = (et_event_count * max(n.value, 1))()
    _check(_lib.et_get_event_counts(g, ctypes.cast(buf, _P), n.value, ctypes.byref(n)), "et_get_event_counts")
    return [(r.kind, r.index, r.count) for r in buf[:n.value]]


def et_get_info(g):
    info = et_graph_info()
    _check(_lib.et_get_info(g, ctypes.byref(info)), "et_get_info")
    return {f: getattr(info, f) for f, _ in et_graph_info._fields_}


def et_get_diag(g):
    out = (ctypes.c_int32 * 8)()
    _check(_lib.et_get_diag(g, out), "et_get_diag")
    return list(out)


def et_destroy_graph(g):
    _lib.et_destroy_graph(g)


def et_status_str(s):
    return _lib.et_status_str(s).decode()
