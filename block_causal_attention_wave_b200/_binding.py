"""ctypes binding of libwave.so: argument marshalling only.

Every computation (scheduling, page allocation, key tables, the append and
attention kernels) happens inside the C library; this module turns Python
values and torch tensors into the plain pointers and sizes the C ABI takes.
There is no fallback: if the library is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwave.so")

OK = 0
ERR_ARG, ERR_MISSING_KV, ERR_NO_PAGES, ERR_CUDA = -1, -2, -3, -4
ERR_TIMEOUT, ERR_EXISTS, ERR_CAPACITY, ERR_UNSUPPORTED = -5, -6, -7, -8
POLICIES = {"clean": 0, "same": 1, "progressive": 2}
PAGE_TOKENS = 128
PREFIX_CHUNK = -1
MAX_NODES = 64
MAX_PAGES_PER_ROUND = 7168

_lib = None


class WaveError(RuntimeError):
    def __init__(self, code: int, detail: str):
        super().__init__(f"wave error {code}: {detail}")
        self.code = code


class Node(ctypes.Structure):
    _fields_ = [("chunk", ctypes.c_int32), ("level", ctypes.c_int32)]


class Rope(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int32), ("rows", ctypes.c_int32), ("cols", ctypes.c_int32),
                ("base", ctypes.c_float)]


ACT_NONE, ACT_GELU_TANH = 0, 1
KV_BF16, KV_FP8_E4M3 = 0, 1


class Transfer(ctypes.Structure):
    _fields_ = [("chunk", ctypes.c_int32), ("level", ctypes.c_int32), ("src", ctypes.c_int32),
                ("dst", ctypes.c_int32)]


class KVConfig(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("tokens_per_chunk", ctypes.c_int32), ("num_levels", ctypes.c_int32),
                ("window", ctypes.c_int32), ("prefix_tokens", ctypes.c_int32),
                ("pool", ctypes.c_void_p), ("pool_bytes", ctypes.c_uint64),
                ("kv_format", ctypes.c_int32)]


_SIGS = {
    "wave_kv_create": (ctypes.c_int, [ctypes.POINTER(KVConfig), ctypes.POINTER(ctypes.c_void_p)]),
    "wave_kv_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "wave_kv_scale_offset": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64)]),
    "wave_kv_pool_layout": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64),
                                           ctypes.POINTER(ctypes.c_int64),
                                           ctypes.POINTER(ctypes.c_int32)]),
    "wave_kv_alloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32]),
    "wave_kv_append": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                      ctypes.c_void_p]),
    "wave_kv_release": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32]),
    "wave_kv_free_pages": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)]),
    "wave_kv_entry_pages": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                                           ctypes.POINTER(ctypes.c_int32)]),
    "wave_gather_table": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(Node), ctypes.c_int32,
                                         ctypes.c_int32, ctypes.POINTER(ctypes.c_int32),
                                         ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                                         ctypes.POINTER(ctypes.c_int32)]),
    "wave_round_attn": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(Node), ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p]),
    "wave_round_attn_static_scratch": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(Node),
                                                      ctypes.c_int32, ctypes.c_int32,
                                                      ctypes.c_void_p, ctypes.c_void_p,
                                                      ctypes.c_void_p]),
    "wave_round_attn_split": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(Node), ctypes.c_int32,
                                             ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64,
                                             ctypes.c_void_p]),
    "wave_round_attn_split_workspace": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(Node),
                                                       ctypes.c_int32, ctypes.c_int32,
                                                       ctypes.c_int32,
                                                       ctypes.POINTER(ctypes.c_uint64),
                                                       ctypes.POINTER(ctypes.c_int32)]),
    "wave_kv_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "wave_kv_set_wait_limit": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_uint64]),
    "wave_qkv_append": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "wave_qkv_append_round": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(Node), ctypes.c_int32,
                                             ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                             ctypes.POINTER(Rope), ctypes.c_void_p,
                                             ctypes.c_void_p]),
    "wave_linear": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                   ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                                   ctypes.c_void_p, ctypes.c_void_p]),
    "wave_kv_append_batch": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(Node),
                                            ctypes.POINTER(ctypes.c_void_p),
                                            ctypes.POINTER(ctypes.c_void_p),
                                            ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p]),
    "wave_kv_last_launch_clock": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.POINTER(ctypes.c_int64),
                                                 ctypes.POINTER(ctypes.c_int64)]),
    "wave_schedule": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.POINTER(Node), ctypes.c_int32,
                                     ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                                     ctypes.POINTER(ctypes.c_int32),
                                     ctypes.POINTER(ctypes.c_int32)]),
    "wave_schedule_last_read": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_int32, ctypes.POINTER(Node),
                                               ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]),
    "wave_wp_transfers": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                         ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                         ctypes.POINTER(Transfer), ctypes.c_int32,
                                         ctypes.POINTER(ctypes.c_int32)]),
    "wave_wp_rank_last_read": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.POINTER(Node), ctypes.c_int32,
                                              ctypes.POINTER(ctypes.c_int32)]),
    "wave_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "wave_last_error_detail": (ctypes.c_char_p, []),
}


def load(path: str = None) -> ctypes.CDLL:
    """Load libwave.so (once). Raises if it has not been built.

    The library next to this file is used unless ``path`` or the environment
    variable WAVE_LIBRARY names another build of it.
    """
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("WAVE_LIBRARY") or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m block_causal_attention_wave_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def exported_symbols():
    return list(_SIGS)


def _check(rc: int):
    if rc != OK:
        detail = _lib.wave_last_error_detail().decode() or _lib.wave_strerror(rc).decode()
        raise WaveError(rc, detail)


def _policy(policy) -> int:
    return POLICIES[policy] if isinstance(policy, str) else int(policy)


def _nodes(active):
    arr = (Node * max(1, len(active)))()
    for i, (c, l) in enumerate(active):
        arr[i].chunk, arr[i].level = int(c), int(l)
    return arr


def _stream_handle(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def schedule(B: int, K: int, policy="progressive", window: int = 0):
    """Rounds of (chunk, level) nodes, as computed by the library."""
    lib = load()
    nn, nr = ctypes.c_int32(0), ctypes.c_int32(0)
    rc = lib.wave_schedule(B, K, _policy(policy), window, None, 0, None, 0,
                           ctypes.byref(nn), ctypes.byref(nr))
    if rc not in (OK, ERR_CAPACITY):
        _check(rc)
    nodes = (Node * nn.value)()
    offs = (ctypes.c_int32 * (nr.value + 1))()
    _check(lib.wave_schedule(B, K, _policy(policy), window, nodes, nn.value, offs, nr.value + 1,
                             ctypes.byref(nn), ctypes.byref(nr)))
    return [[(nodes[i].chunk, nodes[i].level) for i in range(offs[t], offs[t + 1])]
            for t in range(nr.value)]


def last_read_rounds(B: int, K: int, policy="progressive", window: int = 0, nodes=None):
    """Dict (chunk, level) -> last round reading that entry, from the library."""
    lib = load()
    if nodes is None:
        nodes = [n for r in schedule(B, K, policy, window) for n in r]
    arr = _nodes(nodes)
    out = (ctypes.c_int32 * max(1, len(nodes)))()
    _check(lib.wave_schedule_last_read(B, K, _policy(policy), window, arr, len(nodes), out))
    return {tuple(n): out[i] for i, n in enumerate(nodes)}


def wp_transfers(B: int, K: int, policy, window: int, n_ranks: int, round_index: int):
    """Wave Parallelism pushes of one round: [((chunk, level), src, dst), ...]."""
    lib = load()
    n = ctypes.c_int32(0)
    rc = lib.wave_wp_transfers(B, K, _policy(policy), window, n_ranks, round_index, None, 0,
                               ctypes.byref(n))
    if rc not in (OK, ERR_CAPACITY):
        _check(rc)
    buf = (Transfer * max(1, n.value))()
    _check(lib.wave_wp_transfers(B, K, _policy(policy), window, n_ranks, round_index, buf,
                                 n.value, ctypes.byref(n)))
    return [((t.chunk, t.level), t.src, t.dst) for t in buf[:n.value]]


def wp_rank_last_read(B: int, K: int, policy, window: int, n_ranks: int, rank: int, entries):
    """Dict entry -> last round in which a node of ``rank`` reads it."""
    lib = load()
    arr = _nodes(entries)
    out = (ctypes.c_int32 * max(1, len(entries)))()
    _check(lib.wave_wp_rank_last_read(B, K, _policy(policy), window, n_ranks, rank, arr,
                                      len(entries), out))
    return {tuple(e): out[i] for i, e in enumerate(entries)}


class KVCache:
    """Handle on a paged (chunk, level) K/V pool.

    ``pool`` is a caller-owned CUDA uint8 tensor (kept alive by this object).
    With ``pool=None`` the handle is host-only: allocation and tables work,
    kernels do not; ``pool_bytes`` then sets the page count.
    """

    def __init__(self, heads, head_dim, tokens_per_chunk, num_levels, window=0,
                 prefix_tokens=0, pool=None, pool_bytes=None, kv_format=0):
        self.lib = load()
        self.heads, self.head_dim = heads, head_dim
        self.tokens, self.levels = tokens_per_chunk, num_levels
        self.window, self.prefix_tokens = window, prefix_tokens
        self.pool = pool
        if pool is not None:
            pool_bytes = pool.numel() * pool.element_size()
            ptr = pool.data_ptr()
        else:
            ptr = None
        cfg = KVConfig(heads, head_dim, tokens_per_chunk, num_levels, window, prefix_tokens,
                       ptr, int(pool_bytes), int(kv_format))
        self.kv_format = int(kv_format)
        h = ctypes.c_void_p()
        _check(self.lib.wave_kv_create(ctypes.byref(cfg), ctypes.byref(h)))
        self.h = h

    @staticmethod
    def page_bytes(heads, head_dim, kv_format=0) -> int:
        """Bytes of one page (an FP8 pool also keeps 2 H float32 scales per page)."""
        return 2 * heads * PAGE_TOKENS * head_dim * (1 if kv_format == KV_FP8_E4M3 else 2)

    def scale_offset(self) -> int:
        """Byte offset of an FP8 pool's scale table, float32 [max_pages][2][H]."""
        off = ctypes.c_int64()
        _check(self.lib.wave_kv_scale_offset(self.h, ctypes.byref(off)))
        return off.value

    def close(self):
        if getattr(self, "h", None):
            self.lib.wave_kv_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def layout(self):
        pb, off, mp = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
        _check(self.lib.wave_kv_pool_layout(self.h, ctypes.byref(pb), ctypes.byref(off),
                                            ctypes.byref(mp)))
        return pb.value, off.value, mp.value

    def alloc(self, chunk, level, ntokens=None):
        n = self.tokens if ntokens is None else ntokens
        _check(self.lib.wave_kv_alloc(self.h, chunk, level, n))

    def append(self, chunk, level, K, V, stream=None):
        n = K.shape[0]
        _check(self.lib.wave_kv_append(self.h, chunk, level, ctypes.c_void_p(K.data_ptr()),
                                       ctypes.c_void_p(V.data_ptr()), n, _stream_handle(stream)))

    def append_batch(self, entries, Ks, Vs, stream=None):
        """Append several entries with one kernel launch; pages are taken in
        list order, as the same appends one by one would take them."""
        n = len(entries)
        if not (len(Ks) == len(Vs) == n):
            raise ValueError("one K and one V per entry")
        ptr = ctypes.c_void_p * max(n, 1)
        ks = ptr(*[K.data_ptr() for K in Ks])
        vs = ptr(*[V.data_ptr() for V in Vs])
        nt = (ctypes.c_int32 * max(n, 1))(*[K.shape[0] for K in Ks])
        _check(self.lib.wave_kv_append_batch(self.h, n, _nodes(entries), ks, vs, nt,
                                             _stream_handle(stream)))

    def qkv_append(self, chunk, level, X, W, Q, stream=None):
        """Project X [T][C] with W [3 H d][C] into Q (written to ``Q``, [T][H][d])
        and the new entry's K/V pages, in one kernel."""
        _check(self.lib.wave_qkv_append(self.h, chunk, level, ctypes.c_void_p(X.data_ptr()),
                                        X.shape[0], X.shape[1], ctypes.c_void_p(W.data_ptr()),
                                        ctypes.c_void_p(Q.data_ptr()), _stream_handle(stream)))
        return Q

    def qkv_append_round(self, nodes, X, W, Q, rope=None, stream=None):
        """Project the round's nodes (X [n T][C], node i at rows i T) with W
        [3 H d][C] into Q ([n T][H][d]) and each node's new K/V pages, Q and K
        turned by ``rope`` = (frames, rows, cols[, base]) or not (None); one
        kernel launch."""
        r = None
        if rope is not None:
            f, rr, c = rope[:3]
            base = rope[3] if len(rope) > 3 else 10000.0
            r = ctypes.byref(Rope(f, rr, c, base))
        _check(self.lib.wave_qkv_append_round(
            self.h, _nodes(nodes), len(nodes), ctypes.c_void_p(X.data_ptr()), X.shape[1],
            ctypes.c_void_p(W.data_ptr()), r, ctypes.c_void_p(Q.data_ptr()),
            _stream_handle(stream)))
        return Q

    def linear(self, A, W, Y, R=None, act=ACT_NONE, stream=None):
        """Y [M][N] = act(A W^T) (+ R) on the tensor cores; A [M][K], W [N][K]."""
        M, K = A.shape[0], A.numel() // A.shape[0]
        N = W.shape[0]
        _check(self.lib.wave_linear(self.h, ctypes.c_void_p(A.data_ptr()), M, K,
                                    ctypes.c_void_p(W.data_ptr()), N,
                                    ctypes.c_void_p(R.data_ptr()) if R is not None else None,
                                    int(act), ctypes.c_void_p(Y.data_ptr()),
                                    _stream_handle(stream)))
        return Y

    def release(self, chunk, level):
        _check(self.lib.wave_kv_release(self.h, chunk, level))

    def entry_pages(self, chunk, level):
        """Page ids of entry (chunk, level), in token order."""
        n = ctypes.c_int32()
        rc = self.lib.wave_kv_entry_pages(self.h, chunk, level, None, 0, ctypes.byref(n))
        if rc not in (OK, ERR_CAPACITY):
            _check(rc)
        buf = (ctypes.c_int32 * max(1, n.value))()
        _check(self.lib.wave_kv_entry_pages(self.h, chunk, level, buf, n.value, ctypes.byref(n)))
        return list(buf[:n.value])

    def free_pages(self) -> int:
        n = ctypes.c_int32()
        _check(self.lib.wave_kv_free_pages(self.h, ctypes.byref(n)))
        return n.value

    def gather_table(self, active, policy):
        """Per node, a list of (page id, valid tokens) in key order."""
        nodes = _nodes(active)
        n = ctypes.c_int32()
        rc = self.lib.wave_gather_table(self.h, nodes, len(active), _policy(policy), None, None, 0,
                                        ctypes.byref(n))
        if rc not in (OK, ERR_CAPACITY):
            _check(rc)
        rows = (ctypes.c_int32 * (2 * max(1, n.value)))()
        offs = (ctypes.c_int32 * (len(active) + 1))()
        _check(self.lib.wave_gather_table(self.h, nodes, len(active), _policy(policy), rows, offs,
                                          n.value, ctypes.byref(n)))
        return [[(rows[2 * r], rows[2 * r + 1]) for r in range(offs[i], offs[i + 1])]
                for i in range(len(active))]

    def round_attn(self, active, policy, Q, O, stream=None):
        """O[i*T:(i+1)*T] = attention of active node i over its key list."""
        nodes = _nodes(active)
        _check(self.lib.wave_round_attn(self.h, nodes, len(active), _policy(policy),
                                        ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(O.data_ptr()),
                                        _stream_handle(stream)))
        return O

    def split_workspace(self, active, policy, splits=0):
        """(bytes, ranges per item) that round_attn_split needs."""
        b, ns = ctypes.c_uint64(0), ctypes.c_int32(0)
        _check(self.lib.wave_round_attn_split_workspace(self.h, _nodes(active), len(active),
                                                        _policy(policy), int(splits),
                                                        ctypes.byref(b), ctypes.byref(ns)))
        return b.value, ns.value

    def round_attn_split(self, active, policy, Q, O, workspace=None, splits=0, stream=None):
        """round_attn with key lists cut into ranges (0 = automatic count);
        ``workspace`` is a CUDA tensor of at least split_workspace() bytes."""
        ptr = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
        nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        _check(self.lib.wave_round_attn_split(self.h, _nodes(active), len(active),
                                              _policy(policy), int(splits),
                                              ctypes.c_void_p(Q.data_ptr()),
                                              ctypes.c_void_p(O.data_ptr()), ptr, nbytes,
                                              _stream_handle(stream)))
        return O

    def round_attn_static_scratch(self, active, policy, Q, O, stream=None):
        """round_attn whose work-queue counter lives in the library's static
        device array instead of the pool header (no per-call scratch)."""
        nodes = _nodes(active)
        _check(self.lib.wave_round_attn_static_scratch(
            self.h, nodes, len(active), _policy(policy), ctypes.c_void_p(Q.data_ptr()),
            ctypes.c_void_p(O.data_ptr()), _stream_handle(stream)))
        return O

    def status(self, stream=None):
        """Synchronise and raise WaveError if a kernel timed out."""
        _check(self.lib.wave_kv_status(self.h, _stream_handle(stream)))

    def set_wait_limit(self, ns: int = 0):
        """Bound on one device wait of later launches (ns; 0 = default 2 s)."""
        _check(self.lib.wave_kv_set_wait_limit(self.h, int(ns)))

    def last_launch_clock(self, stream=None):
        """(SM cycles, nanoseconds) of the last attention launch's first CTA;
        cycles / ns is the SM clock in GHz that the launch ran at."""
        cyc, ns = ctypes.c_int64(0), ctypes.c_int64(0)
        _check(self.lib.wave_kv_last_launch_clock(self.h, _stream_handle(stream),
                                                  ctypes.byref(cyc), ctypes.byref(ns)))
        return cyc.value, ns.value
