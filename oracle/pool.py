"""The oracle over ranges of view rows in worker processes -- TEST INFRASTRUCTURE ONLY.

Only tests/ and the CPU-baseline legs of bench.py use this module.  It runs the
unchanged single-threaded oracle (oracle_amax, oracle_quantize_rows,
oracle_rht_view, oracle_quantize_rotated) on contiguous ranges of view rows in
separate processes and assembles the pieces.  Each view row's codes and
scales depend only on that row, the tensor amax and the seed (the random
streams are indexed by the full view's element and block numbers), and the
tensor amax is a maximum, so the assembled result is exactly the one-process
result.  Inputs and outputs are shared through memory-mapped files in a
temporary directory; workers are started with `spawn` (never forked from a
process that may already hold a CUDA context).
"""
import concurrent.futures
import ctypes
import multiprocessing
import os
import shutil
import tempfile

import numpy as np


def host_cores() -> int:
    """CPU cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ worker side
def _lib():
    import oracle
    return oracle.lib()


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _open(path, dtype, shape, mode):
    return np.memmap(path, dtype=dtype, mode=mode, shape=tuple(shape))


def _w_ready():
    _lib()
    return os.getpid()


def _w_amax(xpath, shape, layout, g, seed, c0, c1):
    """Oracle amax of the view rows held by x[:, c0:c1] (transposed) or x[c0:c1] (row-wise)."""
    x = _open(xpath, np.uint16, shape, "r")
    sub = np.ascontiguousarray(x[c0:c1] if layout == 0 else x[:, c0:c1])
    rows, cols = sub.shape
    a = np.zeros(1, dtype=np.float32)
    st = _lib().oracle_amax(_ptr(sub), rows, cols, cols, layout, g, seed, _ptr(a))
    if st:
        raise RuntimeError(f"oracle_amax status {st}")
    return float(a[0])


def _w_quantize(xpath, shape, layout, mode, g, seed, amax, b, e, cpath, spath, vr, vc):
    x = _open(xpath, np.uint16, shape, "r")
    codes = _open(cpath, np.uint8, (vr, vc // 2), "r+")
    scales = _open(spath, np.uint8, (vr, vc // 16), "r+")
    rows, cols = shape
    a = np.array([amax], dtype=np.float32)
    gs = np.zeros(1, dtype=np.float32)
    st = _lib().oracle_quantize_rows(_ptr(x), rows, cols, cols, layout, mode, g, seed, _ptr(a), b, e,
                                     _ptr(codes), _ptr(scales), _ptr(gs))
    if st:
        raise RuntimeError(f"oracle_quantize_rows status {st}")
    codes.flush()
    scales.flush()
    return float(gs[0])


def _w_rht_view(xpath, shape, layout, g, seed, c0, c1, zpath, vr, vc):
    """Rotated view rows c0..c1 (row-wise: x rows; transposed: x columns)."""
    x = _open(xpath, np.uint16, shape, "r")
    z = _open(zpath, np.float32, (vr, vc), "r+")
    sub = np.ascontiguousarray(x[c0:c1] if layout == 0 else x[:, c0:c1])
    rows, cols = sub.shape
    out = np.empty((c1 - c0, vc), dtype=np.float32)
    st = _lib().oracle_rht_view(_ptr(sub), rows, cols, cols, layout, g, seed, _ptr(out))
    if st:
        raise RuntimeError(f"oracle_rht_view status {st}")
    z[c0:c1] = out
    z.flush()
    return c1 - c0


def _w_quantize_rotated(zpath, vr, vc, mode, seed, amax, b, e, cpath, spath):
    z = _open(zpath, np.float32, (vr, vc), "r")
    codes = _open(cpath, np.uint8, (vr, vc // 2), "r+")
    scales = _open(spath, np.uint8, (vr, vc // 16), "r+")
    zz = np.ascontiguousarray(z[b:e])
    c = np.zeros((e - b, vc // 2), dtype=np.uint8)
    s = np.zeros((e - b, vc // 16), dtype=np.uint8)
    gs = np.zeros(1, dtype=np.float32)
    st = _lib().oracle_quantize_rotated(_ptr(zz), b, e - b, vc, mode, seed, ctypes.c_float(amax), _ptr(c), _ptr(s),
                                        _ptr(gs))
    if st:
        raise RuntimeError(f"oracle_quantize_rotated status {st}")
    codes[b:e] = c
    scales[b:e] = s
    codes.flush()
    scales.flush()
    return float(gs[0])


# ------------------------------------------------------------------ caller side
def _scratch_dir(min_free=16 << 30):
    """A RAM-backed directory for the shared files when one has room, else the
    default temporary directory."""
    try:
        st = os.statvfs("/dev/shm")
        if st.f_bavail * st.f_frsize >= min_free:
            return "/dev/shm"
    except OSError:
        pass
    return None



class OraclePool:
    """A pool of spawn-started worker processes running the oracle on row ranges.

    with OraclePool() as p:
        a = p.amax(xb, layout, g, seed)
        codes, scales, gs = p.quantize(xb, layout, mode, g, seed, a)
    """

    def __init__(self, workers: int = 0):
        self.workers = workers if workers > 0 else host_cores()
        self._dir = tempfile.mkdtemp(prefix="oracle_pool_", dir=_scratch_dir())
        self._n = 0
        ctx = multiprocessing.get_context("spawn")
        self._ex = concurrent.futures.ProcessPoolExecutor(max_workers=self.workers, mp_context=ctx)
        # start every worker and load the oracle in it now, outside any timing
        list(self._ex.map(_w_ready_n, range(self.workers)))

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def close(self):
        if self._ex is not None:
            self._ex.shutdown(wait=True, cancel_futures=True)
            self._ex = None
        if self._dir and os.path.isdir(self._dir):
            shutil.rmtree(self._dir, ignore_errors=True)
            self._dir = None

    # files -----------------------------------------------------------------
    def _path(self, tag):
        self._n += 1
        return os.path.join(self._dir, f"{tag}_{self._n}.bin")

    def put(self, a):
        """Share an input array with the workers once; the handle can be
        passed to the methods below in place of the array (saves writing
        the same tensor again for every call on it)."""
        return SharedArray(self._share(a, "in"), np.ascontiguousarray(a).dtype, np.shape(a))

    def _input(self, a, dtype, tag):
        """(path, shape, owned) of an input given as an array or a SharedArray."""
        if isinstance(a, SharedArray):
            return a.path, a.shape, False
        a = np.ascontiguousarray(a, dtype=dtype)
        return self._share(a, tag), a.shape, True

    def _share(self, a, tag):
        a = np.ascontiguousarray(a)
        path = self._path(tag)
        m = np.memmap(path, dtype=a.dtype, mode="w+", shape=a.shape)
        m[...] = a
        m.flush()
        del m
        return path

    def _zeros(self, dtype, shape, tag):
        path = self._path(tag)
        m = np.memmap(path, dtype=dtype, mode="w+", shape=tuple(shape))
        m.flush()
        del m
        return path

    def _collect(self, path, dtype, shape):
        m = np.memmap(path, dtype=dtype, mode="r", shape=tuple(shape))
        out = np.array(m)
        del m
        os.unlink(path)
        return out

    def _ranges(self, n, align=1):
        """Split 0..n into about 4 pieces per worker, boundaries multiples of align."""
        pieces = max(1, min(n // max(align, 1), 4 * self.workers))
        edges = sorted(set([0, n] + [min(n, (n * i // pieces) // align * align) for i in range(1, pieces)]))
        return [(edges[i], edges[i + 1]) for i in range(len(edges) - 1) if edges[i + 1] > edges[i]]

    # the oracle, in pieces ---------------------------------------------------
    def amax(self, x_bits, layout, g, seed):
        """oracle.amax of the whole view: the largest of the pieces' amaxes."""
        xpath, (rows, cols), owned = self._input(x_bits, np.uint16, "x")
        if rows * cols == 0:
            if owned:
                os.unlink(xpath)
            return 0.0
        # row-wise: pieces of x rows; transposed: pieces of x columns (whole
        # view rows), 8-aligned as the transposed layout requires
        n = rows if layout == 0 else cols
        futs = [self._ex.submit(_w_amax, xpath, (rows, cols), layout, g, seed, b, e)
                for b, e in self._ranges(n, 1 if layout == 0 else 8)]
        a = max(f.result() for f in futs)
        if owned:
            os.unlink(xpath)
        return a

    def quantize(self, x_bits, layout, mode, g, seed, amax_in, row_range=None):
        """oracle.quantize(x_bits, layout, mode, g, seed, amax_in, row_range) in pieces."""
        xpath, (rows, cols), owned = self._input(x_bits, np.uint16, "x")
        vr, vc = (rows, cols) if layout == 0 else (cols, rows)
        b0, e0 = (0, vr) if row_range is None else row_range
        cpath = self._zeros(np.uint8, (vr, vc // 2), "codes")
        spath = self._zeros(np.uint8, (vr, vc // 16), "scales")
        futs = [self._ex.submit(_w_quantize, xpath, (rows, cols), layout, mode, g, seed, float(amax_in),
                                b0 + b, b0 + e, cpath, spath, vr, vc) for b, e in self._ranges(e0 - b0)]
        gs = [f.result() for f in futs]
        if owned:
            os.unlink(xpath)
        codes = self._collect(cpath, np.uint8, (vr, vc // 2))
        scales = self._collect(spath, np.uint8, (vr, vc // 16))
        return codes, scales, gs[0] if gs else _global_scale(amax_in, mode)

    def rht_view(self, x_bits, layout, g, seed):
        """oracle.rht_view in pieces of view rows."""
        xpath, (rows, cols), owned = self._input(x_bits, np.uint16, "x")
        vr, vc = (rows, cols) if layout == 0 else (cols, rows)
        zpath = self._zeros(np.float32, (vr, vc), "z")
        futs = [self._ex.submit(_w_rht_view, xpath, (rows, cols), layout, g, seed, b, e, zpath, vr, vc)
                for b, e in self._ranges(vr, 1 if layout == 0 else 8)]
        for f in futs:
            f.result()
        if owned:
            os.unlink(xpath)
        return self._collect(zpath, np.float32, (vr, vc))

    def quantize_rotated(self, z, mode, seed, amax):
        """oracle.quantize_rotated of a whole rotated view, in pieces of rows."""
        z = np.ascontiguousarray(z, dtype=np.float32)
        vr, vc = z.shape
        zpath = self._share(z, "z")
        cpath = self._zeros(np.uint8, (vr, vc // 2), "codes")
        spath = self._zeros(np.uint8, (vr, vc // 16), "scales")
        futs = [self._ex.submit(_w_quantize_rotated, zpath, vr, vc, mode, seed, float(amax), b, e, cpath, spath)
                for b, e in self._ranges(vr)]
        gs = [f.result() for f in futs]
        os.unlink(zpath)
        codes = self._collect(cpath, np.uint8, (vr, vc // 2))
        scales = self._collect(spath, np.uint8, (vr, vc // 16))
        return codes, scales, gs[0] if gs else _global_scale(amax, mode)


class SharedArray:
    """An input array already written for the workers (OraclePool.put)."""

    def __init__(self, path, dtype, shape):
        self.path, self.dtype, self.shape = path, dtype, tuple(shape)


def _w_ready_n(_):
    return _w_ready()


def _global_scale(amax, mode):
    import oracle
    return oracle.global_scale(amax, mode)
