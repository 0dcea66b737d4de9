"""Python binding of the B200 e-means library (libemeans.so, C ABI in include/emeans.h).

Argument marshalling only: every step of the method runs in the library's CUDA
kernels. Functions keep the ABI's names; `Model` wraps a handle for convenience
and takes torch tensors (or raw pointers) for X and the outputs.

Importing fails loudly if libemeans.so has not been built (python
mini_ema_means_b200/build.py); there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libemeans.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python mini_ema_means_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

# ---- status codes and options (mirrors include/emeans.h) ----
EM_OK = 0
EM_E_INVAL = -1
EM_E_NOMEM = -2
EM_E_CUDA = -3
EM_E_BOUNDS = -4
EM_E_TIMEOUT = -5
EM_E_NONFINITE = -6
EM_E_STATE = -7
EM_E_NODEVICE = -8
EM_E_COMM = -9

EM_OPT_BATCH_SIZE = 1
EM_OPT_ALPHA0 = 2
EM_OPT_UNUSED_THRESHOLD = 3
EM_OPT_REVIVAL = 4
EM_OPT_FINALIZE = 5
EM_OPT_LAW = 6
EM_OPT_INPUT_DTYPE = 7
EM_OPT_CHECK_FINITE = 8
EM_OPT_WAIT_LIMIT_MS = 9
EM_OPT_AUTO_REVIVE = 10
EM_OPT_CAPTURE_LABELS = 11
EM_OPT_GRAPHS = 12
EM_OPT_ASSIGN_KERNEL = 13
EM_OPT_PROFILE = 14
EM_OPT_EXACT_TIES = 15
EM_OPT_SPHERICAL = 16
EM_OPT_PREFETCH = 17
EM_OPT_SEARCH_FORMAT = 18
EM_OPT_PDL = 19

EM_PHASE_PREPARE = 0
EM_PHASE_GATHER = 1
EM_PHASE_ASSIGN = 2
EM_PHASE_UPDATE = 3
EM_PHASE_REVIVE = 4
EM_PHASE_FINALIZE = 5
EM_NPHASES = 6
PHASE_NAMES = ("prepare", "gather", "assign", "update", "revive", "finalize")

EM_NOALLOC_MAX_ROWS = 524288
EM_NOALLOC_MAX_K = 65536
EM_NOALLOC_MAX_KD = 4194304

EM_REVIVE_NONE = 0
EM_REVIVE_SPLIT = 1
EM_REVIVE_RESAMPLE = 2

REVIVAL_MODES = {"none": EM_REVIVE_NONE, "split": EM_REVIVE_SPLIT, "resample": EM_REVIVE_RESAMPLE}


class em_recipe_t(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("d", ctypes.c_int64),
        ("epochs", ctypes.c_double), ("batch_raw", ctypes.c_double),
        ("batch_size", ctypes.c_int64), ("alpha0", ctypes.c_double),
        ("passes", ctypes.c_int64), ("rows_last_pass", ctypes.c_int64),
        ("steps_full_pass", ctypes.c_int64), ("steps_last_pass", ctypes.c_int64),
        ("total_steps", ctypes.c_int64),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class em_stats_t(ctypes.Structure):
    _fields_ = [
        ("steps_done", ctypes.c_int64), ("passes_done", ctypes.c_int64),
        ("rows_assigned", ctypes.c_int64), ("n_splits", ctypes.c_int64),
        ("last_dead", ctypes.c_int64), ("imbalance", ctypes.c_double),
        ("last_alpha", ctypes.c_double),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class em_profile_t(ctypes.Structure):
    _fields_ = [
        ("ms", ctypes.c_double * EM_NPHASES), ("spans", ctypes.c_int64 * EM_NPHASES),
        ("launches", ctypes.c_int64), ("assign_flops", ctypes.c_double),
        ("update_bytes", ctypes.c_double), ("gather_bytes", ctypes.c_double),
    ]

    def as_dict(self):
        return {
            "ms": dict(zip(PHASE_NAMES, list(self.ms))),
            "spans": dict(zip(PHASE_NAMES, list(self.spans))),
            "launches": self.launches, "assign_flops": self.assign_flops,
            "update_bytes": self.update_bytes, "gather_bytes": self.gather_bytes,
        }


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGS = {
    "em_last_error": (ctypes.c_char_p, []),
    "em_device_count": (ctypes.c_int, []),
    "em_last_error_code": (ctypes.c_int, []),
    "em_fail_allocation": (_I64, [_I64]),
    "em_compute_recipe": (ctypes.c_int, [_I64, _I64, ctypes.c_double, ctypes.c_int, _I64, ctypes.c_double,
                                         ctypes.POINTER(em_recipe_t)]),
    "em_permutation": (ctypes.c_int, [_I64, ctypes.c_uint64, ctypes.c_int, _I64, _P, _I64, _P]),
    "em_dp_schedule": (ctypes.c_int, [_I64, _I64, ctypes.c_double, ctypes.c_int, _I64, ctypes.c_double, _I64, _I64,
                                      _I64, _P, _P, _P, _P]),
    "em_search_schedule": (ctypes.c_int, [_I64, _I64, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                          ctypes.POINTER(ctypes.c_int)]),
    "em_create": (_P, [_I64, _I64, ctypes.c_uint64]),
    "em_destroy": (None, [_P]),
    "em_set_option": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_double]),
    "em_get_option": (ctypes.c_int, [_P, ctypes.c_int, ctypes.POINTER(ctypes.c_double)]),
    "em_set_stream": (ctypes.c_int, [_P, _P]),
    "em_train": (ctypes.c_int, [_P, _P, _I64, ctypes.c_double]),
    "em_begin": (ctypes.c_int, [_P, _P, _I64, ctypes.c_double]),
    "em_step": (ctypes.c_int, [_P, _I64, ctypes.POINTER(_I64)]),
    "em_finalize": (ctypes.c_int, [_P]),
    "em_revive": (ctypes.c_int, [_P]),
    "em_lloyd": (ctypes.c_int, [_P, _P, _I64, _I64]),
    "em_assign": (ctypes.c_int, [_P, _P, _I64, _P, _P]),
    "em_mse": (ctypes.c_int, [_P, _P, _I64, ctypes.POINTER(ctypes.c_double)]),
    "em_centroids": (ctypes.c_int, [_P, _P]),
    "em_labels": (ctypes.c_int, [_P, _P]),
    "em_recipe": (ctypes.c_int, [_P, ctypes.POINTER(em_recipe_t)]),
    "em_stats": (ctypes.c_int, [_P, ctypes.POINTER(em_stats_t)]),
    "em_obj": (ctypes.c_int, [_P, _P, _I64, ctypes.POINTER(_I64)]),
    "em_get_state": (ctypes.c_int, [_P, _P, _P, _P, ctypes.POINTER(_I64)]),
    "em_set_state": (ctypes.c_int, [_P, _P, _P, _P, _I64]),
    "em_last_batch": (ctypes.c_int, [_P, _P, _P, _P, ctypes.POINTER(_I64)]),
    "em_profile": (ctypes.c_int, [_P, ctypes.POINTER(em_profile_t), ctypes.c_int]),
    "em_assign_noalloc": (ctypes.c_int, [_P, _I64, _I64, _P, _I64, _P, _P, _P]),
    "em_sync": (ctypes.c_int, [_P]),
    "em_selftest": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_double]),
    "em_fp8_converter": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_float)]),
    "em_dp_unique_id": (ctypes.c_int, [_P]),
    "em_dp_init": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, _P]),
    "em_dp_world": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
}

EM_NCCL_ID_BYTES = 128


def dp_unique_id() -> bytes:
    """A fresh communicator id for em_dp_init (rank 0 makes it, the others receive it)."""
    buf = ctypes.create_string_buffer(EM_NCCL_ID_BYTES)
    check(em_dp_unique_id(ctypes.cast(buf, ctypes.c_void_p)), "em_dp_unique_id")
    return buf.raw

for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args
    globals()[_name] = _fn

ABI_FUNCTIONS = tuple(_SIGS)


class EmeansError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = em_last_error().decode(errors="replace")
        super().__init__(f"{where} failed with status {code}: {msg}")
        self.code = code


def check(rc: int, where: str = "call") -> None:
    if rc != EM_OK:
        raise EmeansError(rc, where)


def _ptr(x):
    """Address of a tensor / ndarray / raw int (0 for None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def compute_recipe(n, k, epochs, law=0, batch_size=0, alpha0=0.0) -> dict:
    r = em_recipe_t()
    check(em_compute_recipe(n, k, float(epochs), int(law), int(batch_size), float(alpha0), ctypes.byref(r)),
          "em_compute_recipe")
    return r.as_dict()


def search_schedule(rows, k, sms):
    """(split, m_full) of the nearest-centroid search for `rows` rows and k
    centroids on `sms` SMs (host code)."""
    split, m_full = ctypes.c_int(), ctypes.c_int()
    check(em_search_schedule(int(rows), int(k), int(sms), ctypes.byref(split), ctypes.byref(m_full)),
          "em_search_schedule")
    return split.value, m_full.value


def permutation(n, seed, stream, which, idx):
    """pi(idx) of the library's keyed bijection (host code; idx: int64 ndarray)."""
    import numpy as np

    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty_like(idx)
    check(em_permutation(n, seed, stream, which, idx.ctypes.data, len(idx), out.ctypes.data), "em_permutation")
    return out


def fail_allocation(nth: int) -> int:
    """Makes the library's nth device allocation from now on fail as a failed
    cudaMalloc does (nth <= 0: off); returns the allocations attempted since the
    previous call (host code)."""
    return int(em_fail_allocation(int(nth)))


def dp_schedule(n_local, k, epochs, world, rank, count, law=0, batch_size=0, alpha0=0.0):
    """The rows rank `rank` of `world` takes at each of the first `count` steps of a
    data-parallel run (host code): arrays pass, first, rows, key (int64)."""
    import numpy as np

    out = [np.empty(count, dtype=np.int64) for _ in range(4)]
    check(em_dp_schedule(n_local, k, epochs, law, batch_size, alpha0, world, rank, count,
                         *(o.ctypes.data for o in out)), "em_dp_schedule")
    return tuple(out)


def exchange_dp_id(group=None):
    """(world, rank, id): rank 0 of a torch.distributed group makes a communicator id
    and broadcasts it to the group's other ranks."""
    import torch.distributed as dist

    world, rank = dist.get_world_size(group), dist.get_rank(group)
    obj = [dp_unique_id() if rank == 0 else None]
    src = 0 if group is None else dist.get_global_rank(group, 0)
    dist.broadcast_object_list(obj, src=src, group=group)
    return world, rank, obj[0]


class Model:
    """One e-means model (handle owner). X and outputs are torch tensors or pointers."""

    def __init__(self, d: int, k: int, seed: int = 1234, **options):
        h = em_create(int(d), int(k), int(seed))
        if not h:
            raise EmeansError(em_last_error_code() or EM_E_INVAL, "em_create")
        self.h = h
        self.d, self.k, self.seed = int(d), int(k), int(seed)
        for name, value in options.items():
            self.set_option(name, value)

    _OPTS = {
        "batch_size": EM_OPT_BATCH_SIZE, "alpha0": EM_OPT_ALPHA0, "unused_threshold": EM_OPT_UNUSED_THRESHOLD,
        "revival": EM_OPT_REVIVAL, "finalize": EM_OPT_FINALIZE, "law": EM_OPT_LAW,
        "input_dtype": EM_OPT_INPUT_DTYPE, "check_finite": EM_OPT_CHECK_FINITE,
        "wait_limit_ms": EM_OPT_WAIT_LIMIT_MS, "auto_revive": EM_OPT_AUTO_REVIVE,
        "capture_labels": EM_OPT_CAPTURE_LABELS, "graphs": EM_OPT_GRAPHS, "assign_kernel": EM_OPT_ASSIGN_KERNEL,
        "profile": EM_OPT_PROFILE, "exact_ties": EM_OPT_EXACT_TIES, "spherical": EM_OPT_SPHERICAL,
        "prefetch": EM_OPT_PREFETCH, "search_format": EM_OPT_SEARCH_FORMAT, "pdl": EM_OPT_PDL,
    }

    def set_option(self, name, value):
        if name == "revival" and isinstance(value, str):
            value = REVIVAL_MODES[value]
        if name == "search_format" and isinstance(value, str):
            value = {"bf16": 0, "fp8": 1, "e4m3": 1}[value]
        if name == "law" and isinstance(value, str):
            value = {"throughput": 0, "quality": 1, "auto": 2}[value]
        if name == "input_dtype" and not isinstance(value, (int, float)):
            value = 1 if "bfloat16" in str(value) or str(value) == "bf16" else 0
        check(em_set_option(self.h, self._OPTS[name], float(value)), f"em_set_option({name})")

    def get_option(self, name) -> float:
        v = ctypes.c_double()
        check(em_get_option(self.h, self._OPTS[name], ctypes.byref(v)), "em_get_option")
        return v.value

    def _dtype_of(self, X):
        if hasattr(X, "dtype"):
            self.set_option("input_dtype", 1 if "bfloat16" in str(X.dtype) else 0)

    def set_stream(self, stream):
        check(em_set_stream(self.h, stream), "em_set_stream")

    def dp_init(self, group=None):
        """Data-parallel training over the ranks of a torch.distributed group (one
        process per GPU): rank 0 makes the communicator id and the group broadcasts
        it; the library then runs its own NCCL communicator."""
        world, rank, uid = exchange_dp_id(group)
        self.dp_init_id(world, rank, uid)

    def dp_init_id(self, world, rank, uid: bytes):
        """em_dp_init with an id already shared by the caller (every rank calls it)."""
        buf = ctypes.create_string_buffer(bytes(uid), EM_NCCL_ID_BYTES)
        check(em_dp_init(self.h, int(world), int(rank), ctypes.cast(buf, ctypes.c_void_p)), "em_dp_init")

    def fp8_converter(self):
        """(shift, scale) of the fitted FP8 converter: shift as a float32 ndarray of d."""
        import numpy as np

        shift = np.empty(self.d, dtype=np.float32)
        sc = ctypes.c_float()
        check(em_fp8_converter(self.h, shift.ctypes.data, ctypes.byref(sc)), "em_fp8_converter")
        return shift, float(sc.value)

    def selftest(self, which, wait_ms=200.0) -> int:
        """Status of em_selftest (EM_E_TIMEOUT for which=0, EM_E_BOUNDS for which=1)."""
        return int(em_selftest(self.h, int(which), float(wait_ms)))

    def dp_world(self):
        w, r = ctypes.c_int(), ctypes.c_int()
        check(em_dp_world(self.h, ctypes.byref(w), ctypes.byref(r)), "em_dp_world")
        return w.value, r.value

    def train(self, X, n=None, epochs=5.0):
        self._dtype_of(X)
        check(em_train(self.h, _ptr(X), int(n if n is not None else X.shape[0]), float(epochs)), "em_train")

    def begin(self, X, n=None, epochs=5.0):
        self._dtype_of(X)
        check(em_begin(self.h, _ptr(X), int(n if n is not None else X.shape[0]), float(epochs)), "em_begin")
        return self.recipe()

    def step(self, nsteps=1) -> int:
        done = _I64()
        check(em_step(self.h, int(nsteps), ctypes.byref(done)), "em_step")
        return done.value

    def finalize(self):
        check(em_finalize(self.h), "em_finalize")

    def revive(self):
        check(em_revive(self.h), "em_revive")

    def lloyd(self, X, iters, n=None):
        self._dtype_of(X)
        check(em_lloyd(self.h, _ptr(X), int(n if n is not None else X.shape[0]), int(iters)), "em_lloyd")

    def assign(self, X, labels=None, dists=None, n=None):
        self._dtype_of(X)
        check(em_assign(self.h, _ptr(X), int(n if n is not None else X.shape[0]), _ptr(labels), _ptr(dists)),
              "em_assign")

    def mse(self, X, n=None) -> float:
        self._dtype_of(X)
        out = ctypes.c_double()
        check(em_mse(self.h, _ptr(X), int(n if n is not None else X.shape[0]), ctypes.byref(out)), "em_mse")
        return out.value

    def centroids(self, out):
        check(em_centroids(self.h, _ptr(out)), "em_centroids")
        return out

    def labels(self, out):
        check(em_labels(self.h, _ptr(out)), "em_labels")
        return out

    def recipe(self) -> dict:
        r = em_recipe_t()
        check(em_recipe(self.h, ctypes.byref(r)), "em_recipe")
        return r.as_dict()

    def stats(self) -> dict:
        s = em_stats_t()
        check(em_stats(self.h, ctypes.byref(s)), "em_stats")
        return s.as_dict()

    def obj(self):
        import numpy as np

        cnt = _I64()
        check(em_obj(self.h, None, 0, ctypes.byref(cnt)), "em_obj")
        out = np.zeros(max(cnt.value, 1))
        check(em_obj(self.h, out.ctypes.data, cnt.value, ctypes.byref(cnt)), "em_obj")
        return out[:cnt.value]

    def get_state(self, N=None, S=None, c=None) -> int:
        step = _I64()
        check(em_get_state(self.h, _ptr(N), _ptr(S), _ptr(c), ctypes.byref(step)), "em_get_state")
        return step.value

    def set_state(self, N=None, S=None, c=None, step=0):
        check(em_set_state(self.h, _ptr(N), _ptr(S), _ptr(c), int(step)), "em_set_state")

    def last_batch(self, ids=None, labels=None, dists=None) -> int:
        rows = _I64()
        check(em_last_batch(self.h, _ptr(ids), _ptr(labels), _ptr(dists), ctypes.byref(rows)), "em_last_batch")
        return rows.value

    def profile(self, reset=False) -> dict:
        p = em_profile_t()
        check(em_profile(self.h, ctypes.byref(p), int(reset)), "em_profile")
        return p.as_dict()

    def sync(self):
        check(em_sync(self.h), "em_sync")

    def close(self):
        if getattr(self, "h", None):
            em_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
