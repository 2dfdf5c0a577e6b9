"""CPU oracle for int4 KV-cache quantization and decode attention over the
packed int4 cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package.  The product path (the CUDA library and its binding) never
imports it, and it imports nothing from the product path.

The arithmetic lives in ``oracle.c`` (plain C, fp64, explicit d x d rotation
matrix); this module only compiles it with gcc and marshals numpy arrays.
See the header of ``oracle.c`` for the method's sources and the readings
taken where the pages are silent.

Every function here is pinned by ``tests/test_oracle_pins.py`` against facts
the pages or mathematics fix (Sylvester recursion, orthogonality, the
quantizer's half-step bound, exact recovery on the int4 grid, round-half-even
ties, hand-derived byte layouts, closed-form attention cases and brute-force
softmax on tiny inputs; the SRFT variant against numpy's FFT, the Hartley
transform's involution and attention over a cache built exactly on the grid).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_GROUP = 32
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, fp64, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared",
           "-fPIC", "-std=c11", "-Wall", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_hadamard_entry.argtypes = [i32, i32]
    lib.oracle_hadamard_entry.restype = i32
    lib.oracle_rotation_matrix.argtypes = [i32, P, P]
    lib.oracle_rotation_matrix.restype = i32
    lib.oracle_rotate_vector.argtypes = [i32, P, P, P]
    lib.oracle_rotate_vector.restype = None
    lib.oracle_quantize_vector.argtypes = [i32, P, P, P]
    lib.oracle_quantize_vector.restype = None
    lib.oracle_packed_byte_index.argtypes = [i32, i32]
    lib.oracle_packed_byte_index.restype = i64
    lib.oracle_pack_vector.argtypes = [i32, P, P]
    lib.oracle_pack_vector.restype = None
    lib.oracle_unpack_vector.argtypes = [i32, P, P]
    lib.oracle_unpack_vector.restype = None
    lib.oracle_quantize_append.argtypes = [P, P, i32, i32, i32, i32, i32, P, P, P, P, P, P,
                                           i64, i32]
    lib.oracle_quantize_append.restype = i32
    lib.oracle_sdpa_int4_decode.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P, i64, P, P,
                                            f64, P, i32]
    lib.oracle_sdpa_int4_decode.restype = i32
    lib.oracle_exact_attention.argtypes = [P, i32, P, P, i32, i32, i32, i32, i32, i64, P, f64,
                                           P, i32]
    lib.oracle_exact_attention.restype = i32
    lib.oracle_dht_entry.argtypes = [i32, i32, i32]
    lib.oracle_dht_entry.restype = f64
    lib.oracle_srft_matrix.argtypes = [i32, P, P, P]
    lib.oracle_srft_matrix.restype = i32
    lib.oracle_quantize_append_srft.argtypes = [P, P, i32, i32, i32, i32, i32, P, P, P, P, P, P,
                                                P, P, i64, i32]
    lib.oracle_quantize_append_srft.restype = i32
    lib.oracle_sdpa_int4_decode_srft.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P, i64, P,
                                                 P, P, P, f64, P, i32]
    lib.oracle_sdpa_int4_decode_srft.restype = i32
    lib.oracle_lloyd_max_gaussian.argtypes = [i32, P]
    lib.oracle_lloyd_max_gaussian.restype = i32
    lib.oracle_cb_quantize_vector.argtypes = [i32, P, i32, P, P, P]
    lib.oracle_cb_quantize_vector.restype = None
    lib.oracle_cb_pack_vector.argtypes = [i32, i32, P, P]
    lib.oracle_cb_pack_vector.restype = None
    lib.oracle_cb_unpack_vector.argtypes = [i32, i32, P, P]
    lib.oracle_cb_unpack_vector.restype = None
    lib.oracle_quantize_append_cb.argtypes = [P, P, i32, i32, i32, i32, i32, P, P, i32, P, P, P,
                                              P, P, i64, i32]
    lib.oracle_quantize_append_cb.restype = i32
    lib.oracle_sdpa_cb_decode.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, i64, P, P,
                                          f64, P, i32]
    lib.oracle_sdpa_cb_decode.restype = i32
    lib.oracle_uniform_levels.argtypes = [i32, P]
    lib.oracle_uniform_levels.restype = i32
    lib.oracle_uniform_quantize_vector.argtypes = [i32, P, i32, P, P]
    lib.oracle_uniform_quantize_vector.restype = None
    lib.oracle_quantize_append_uniform.argtypes = [P, P, i32, i32, i32, i32, i32, P, P, i32, P, P,
                                                   P, P, i64, i32]
    lib.oracle_quantize_append_uniform.restype = i32
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = i32
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _input_array(x):
    """(array, dtype code): fp32 -> 0; bf16 given as uint16 bit patterns -> 1."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, 0
    if x.dtype == np.uint16:
        return x, 1
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {x.dtype}")


def _signs_array(signs):
    if signs is None:
        return None
    s = np.ascontiguousarray(signs, dtype=np.int8)
    if not np.all(np.abs(s) == 1):
        raise ValueError("signs must be +1/-1")
    return s


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def hadamard_entry(i: int, j: int) -> int:
    return int(_load().oracle_hadamard_entry(i, j))


def rotation_matrix(d: int, signs=None) -> np.ndarray:
    """R = H_d diag(signs) / sqrt(d) (identity when signs is None), fp64 (d, d)."""
    R = np.empty((d, d), dtype=np.float64)
    s = _signs_array(signs)
    if _load().oracle_rotation_matrix(d, _ptr(s), _ptr(R)) != 0:
        raise ValueError("d must be a power of two")
    return R


def rotate(x: np.ndarray, signs=None) -> np.ndarray:
    """fl32(R x) for each row of x (float32, (n, d))."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, d = x.shape
    R = rotation_matrix(d, signs)
    y = np.empty_like(x)
    lib = _load()
    for r in range(n):
        lib.oracle_rotate_vector(d, _ptr(R), _ptr(x[r]), _ptr(y[r]))
    return y


def _lambda_array(lam, d):
    if lam is None:
        return None
    a = np.ascontiguousarray(lam, dtype=np.float32)
    if a.shape != (d,) or not np.all(np.isfinite(a)) or not np.all(a > 0):
        raise ValueError("lambda must be d positive finite float32 values")
    return a


def dht_entry(d: int, k: int, j: int) -> float:
    """Orthonormal discrete Hartley transform entry cas(2 pi k j / d) / sqrt(d)."""
    return float(_load().oracle_dht_entry(d, k, j))


def srft_matrix(d: int, signs=None, lam=None) -> np.ndarray:
    """Store map of the SRFT variant: A = diag(lam) F_d diag(signs), fp64 (d, d)."""
    A = np.empty((d, d), dtype=np.float64)
    if _load().oracle_srft_matrix(d, _ptr(_signs_array(signs)), _ptr(_lambda_array(lam, d)),
                                  _ptr(A)) != 0:
        raise ValueError("d must be positive")
    return A


def srft_rotate(x: np.ndarray, signs=None, lam=None) -> np.ndarray:
    """fl32(A x) for each row of x (float32, (n, d)), A the SRFT store map."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, d = x.shape
    A = srft_matrix(d, signs, lam)
    y = np.empty_like(x)
    lib = _load()
    for r in range(n):
        lib.oracle_rotate_vector(d, _ptr(A), _ptr(x[r]), _ptr(y[r]))
    return y


def quantize_vectors(y: np.ndarray):
    """Group abs-max int4 of already-rotated rows y (float32, (n, d)).

    Returns (codes int8 (n, d), scales float32 (n, d/32)).
    """
    y = np.ascontiguousarray(y, dtype=np.float32)
    n, d = y.shape
    codes = np.empty((n, d), dtype=np.int8)
    scales = np.empty((n, d // _GROUP), dtype=np.float32)
    lib = _load()
    for r in range(n):
        lib.oracle_quantize_vector(d, _ptr(y[r]), _ptr(codes[r]), _ptr(scales[r]))
    return codes, scales


def packed_byte_index(d: int, i: int) -> int:
    return int(_load().oracle_packed_byte_index(d, i))


def pack(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    n, d = codes.shape
    out = np.empty((n, d // 2), dtype=np.uint8)
    lib = _load()
    for r in range(n):
        lib.oracle_pack_vector(d, _ptr(codes[r]), _ptr(out[r]))
    return out


def unpack(packed: np.ndarray, d: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    out = np.empty((n, d), dtype=np.int8)
    lib = _load()
    for r in range(n):
        lib.oracle_unpack_vector(d, _ptr(packed[r]), _ptr(out[r]))
    return out


def empty_cache(B: int, Hkv: int, capacity: int, d: int):
    """Zeroed (k_packed, k_scales, v_packed, v_scales) host arrays."""
    return (np.zeros((B, Hkv, capacity, d // 2), np.uint8),
            np.zeros((B, Hkv, capacity, d // _GROUP), np.float32),
            np.zeros((B, Hkv, capacity, d // 2), np.uint8),
            np.zeros((B, Hkv, capacity, d // _GROUP), np.float32))


def quantize_append(k, v, pos, signs, cache, threads: int = 1) -> None:
    """Quantize k, v ([B][Hkv][n_new][d], fp32 or bf16 bits) into `cache` in place."""
    k, dt = _input_array(k)
    v, dt2 = _input_array(v)
    if dt != dt2 or k.shape != v.shape:
        raise ValueError("k and v must share dtype and shape")
    B, Hkv, n_new, d = k.shape
    kp, ks, vp, vs = cache
    cap = kp.shape[2]
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    s = _signs_array(signs)
    rc = _load().oracle_quantize_append(_ptr(k), _ptr(v), dt, B, Hkv, n_new, d, _ptr(pos),
                                        _ptr(s), _ptr(kp), _ptr(ks), _ptr(vp), _ptr(vs), cap,
                                        threads)
    if rc != 0:
        raise ValueError(f"oracle_quantize_append failed ({rc})")


def quantize_append_srft(k, v, pos, signs, lambda_k, lambda_v, cache, threads: int = 1) -> None:
    """SRFT variant of quantize_append: stored rows are fl32(lambda (.) F (signs (.) x))."""
    k, dt = _input_array(k)
    v, dt2 = _input_array(v)
    if dt != dt2 or k.shape != v.shape:
        raise ValueError("k and v must share dtype and shape")
    B, Hkv, n_new, d = k.shape
    kp, ks, vp, vs = cache
    cap = kp.shape[2]
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    s = _signs_array(signs)
    lk, lv = _lambda_array(lambda_k, d), _lambda_array(lambda_v, d)
    rc = _load().oracle_quantize_append_srft(_ptr(k), _ptr(v), dt, B, Hkv, n_new, d, _ptr(pos),
                                             _ptr(s), _ptr(lk), _ptr(lv), _ptr(kp), _ptr(ks),
                                             _ptr(vp), _ptr(vs), cap, threads)
    if rc != 0:
        raise ValueError(f"oracle_quantize_append_srft failed ({rc})")


def sdpa_int4_decode_srft(q, cache, ctx_lens, signs, lambda_k, lambda_v, attn_scale: float,
                          num_kv_heads: int, threads: int = 1) -> np.ndarray:
    """SRFT variant of sdpa_int4_decode: q_r = F (signs (.) q) / lambda_k,
    o = signs (.) F (o_r / lambda_v); returns (B, Hq, d) fp64."""
    q, qdt = _input_array(q)
    B, Hq, d = q.shape
    kp, ks, vp, vs = [np.ascontiguousarray(a) for a in cache]
    cap = kp.shape[2]
    ctx = np.ascontiguousarray(ctx_lens, dtype=np.int32)
    s = _signs_array(signs)
    lk, lv = _lambda_array(lambda_k, d), _lambda_array(lambda_v, d)
    out = np.empty((B, Hq, d), dtype=np.float64)
    rc = _load().oracle_sdpa_int4_decode_srft(_ptr(q), qdt, B, Hq, num_kv_heads, d, _ptr(kp),
                                              _ptr(ks), _ptr(vp), _ptr(vs), cap, _ptr(ctx),
                                              _ptr(s), _ptr(lk), _ptr(lv), float(attn_scale),
                                              _ptr(out), threads)
    if rc != 0:
        raise ValueError(f"oracle_sdpa_int4_decode_srft failed ({rc})")
    return out


def sdpa_int4_decode(q, cache, ctx_lens, signs, attn_scale: float, num_kv_heads: int,
                     threads: int = 1) -> np.ndarray:
    """fp64 attention of q ([B][Hq][d]) over the packed cache; returns (B, Hq, d) fp64."""
    q, qdt = _input_array(q)
    B, Hq, d = q.shape
    kp, ks, vp, vs = [np.ascontiguousarray(a) for a in cache]
    cap = kp.shape[2]
    ctx = np.ascontiguousarray(ctx_lens, dtype=np.int32)
    s = _signs_array(signs)
    out = np.empty((B, Hq, d), dtype=np.float64)
    rc = _load().oracle_sdpa_int4_decode(_ptr(q), qdt, B, Hq, num_kv_heads, d, _ptr(kp),
                                         _ptr(ks), _ptr(vp), _ptr(vs), cap, _ptr(ctx), _ptr(s),
                                         float(attn_scale), _ptr(out), threads)
    if rc != 0:
        raise ValueError(f"oracle_sdpa_int4_decode failed ({rc})")
    return out


def exact_attention(q, k, v, ctx_lens, attn_scale: float, threads: int = 1) -> np.ndarray:
    """Unquantized fp64 softmax attention (fidelity report only).

    q [B][Hq][d]; k, v [B][Hkv][capacity][d] (fp32 or bf16 bits).
    """
    q, qdt = _input_array(q)
    k, kdt = _input_array(k)
    v, vdt = _input_array(v)
    if kdt != vdt:
        raise ValueError("k and v must share dtype")
    B, Hq, d = q.shape
    Hkv, cap = k.shape[1], k.shape[2]
    ctx = np.ascontiguousarray(ctx_lens, dtype=np.int32)
    out = np.empty((B, Hq, d), dtype=np.float64)
    rc = _load().oracle_exact_attention(_ptr(q), qdt, _ptr(k), _ptr(v), kdt, B, Hq, Hkv, d, cap,
                                        _ptr(ctx), float(attn_scale), _ptr(out), threads)
    if rc != 0:
        raise ValueError(f"oracle_exact_attention failed ({rc})")
    return out


# ------------------------------------------------------------ codebook variant
# AdapTQ's Max-Lloyd codebook indices at 2, 3 or 4 bits per coordinate (see the
# header of oracle.c for the quantizer and the packed layout).

def lloyd_max_gaussian(bits: int) -> np.ndarray:
    """Gaussian Max-Lloyd codebook of 2**bits increasing levels (fp64)."""
    out = np.empty(1 << bits, dtype=np.float64)
    if _load().oracle_lloyd_max_gaussian(bits, _ptr(out)) != 0:
        raise ValueError("bits must be in 1..8")
    return out


def _levels_array(levels, bits):
    c = np.ascontiguousarray(levels, dtype=np.float32)
    if c.shape != (1 << bits,) or not np.all(np.diff(c) > 0):
        raise ValueError("levels must be 2**bits strictly increasing float32 values")
    return c


def cb_row_bytes(d: int, bits: int) -> int:
    return d * bits // 8


def cb_quantize_vectors(y: np.ndarray, bits: int, levels):
    """Codebook indices (uint8 (n, d)) and sigma scales (float32 (n, d/32)) of rotated rows y."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    n, d = y.shape
    c = _levels_array(levels, bits)
    idx = np.empty((n, d), dtype=np.uint8)
    scales = np.empty((n, d // _GROUP), dtype=np.float32)
    lib = _load()
    for r in range(n):
        lib.oracle_cb_quantize_vector(d, _ptr(y[r]), bits, _ptr(c), _ptr(idx[r]), _ptr(scales[r]))
    return idx, scales


def cb_pack(idx: np.ndarray, bits: int) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.uint8)
    n, d = idx.shape
    out = np.empty((n, cb_row_bytes(d, bits)), dtype=np.uint8)
    lib = _load()
    for r in range(n):
        lib.oracle_cb_pack_vector(d, bits, _ptr(idx[r]), _ptr(out[r]))
    return out


def cb_unpack(packed: np.ndarray, d: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    out = np.empty((n, d), dtype=np.uint8)
    lib = _load()
    for r in range(n):
        lib.oracle_cb_unpack_vector(d, bits, _ptr(packed[r]), _ptr(out[r]))
    return out


def empty_cb_cache(B: int, Hkv: int, capacity: int, d: int, bits: int):
    """Zeroed (k_packed, k_scales, v_packed, v_scales) of a codebook cache."""
    rb = cb_row_bytes(d, bits)
    return (np.zeros((B, Hkv, capacity, rb), np.uint8),
            np.zeros((B, Hkv, capacity, d // _GROUP), np.float32),
            np.zeros((B, Hkv, capacity, rb), np.uint8),
            np.zeros((B, Hkv, capacity, d // _GROUP), np.float32))


def quantize_append_cb(k, v, pos, signs, bits: int, levels, cache, threads: int = 1) -> None:
    """Codebook variant of quantize_append (Hadamard rotation with signs, or none)."""
    k, dt = _input_array(k)
    v, dt2 = _input_array(v)
    if dt != dt2 or k.shape != v.shape:
        raise ValueError("k and v must share dtype and shape")
    B, Hkv, n_new, d = k.shape
    kp, ks, vp, vs = cache
    cap = kp.shape[2]
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    s = _signs_array(signs)
    c = _levels_array(levels, bits)
    rc = _load().oracle_quantize_append_cb(_ptr(k), _ptr(v), dt, B, Hkv, n_new, d, _ptr(pos), _ptr(s),
                                           bits, _ptr(c), _ptr(kp), _ptr(ks), _ptr(vp), _ptr(vs), cap,
                                           threads)
    if rc != 0:
        raise ValueError(f"oracle_quantize_append_cb failed ({rc})")


def uniform_levels(bits: int) -> np.ndarray:
    """The decode-side table of a uniform low-bit cache: levels[u] = u - m, m = 2^(bits-1) - 1."""
    out = np.empty(1 << bits, dtype=np.float32)
    if _load().oracle_uniform_levels(bits, _ptr(out)) != 0:
        raise ValueError(f"uniform levels: bits must be 2..4, got {bits}")
    return out


def uniform_quantize_vectors(y: np.ndarray, bits: int):
    """Uniform abs-max indices c + m (uint8 (n, d)) and scales (float32 (n, d/32)) of rotated rows y."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    n, d = y.shape
    idx = np.empty((n, d), dtype=np.uint8)
    scales = np.empty((n, d // _GROUP), dtype=np.float32)
    lib = _load()
    for r in range(n):
        lib.oracle_uniform_quantize_vector(d, _ptr(y[r]), bits, _ptr(idx[r]), _ptr(scales[r]))
    return idx, scales


def quantize_append_uniform(k, v, pos, signs, bits: int, cache, threads: int = 1) -> None:
    """Uniform low-bit variant of quantize_append into a codebook-layout cache."""
    k, dt = _input_array(k)
    v, dt2 = _input_array(v)
    if dt != dt2 or k.shape != v.shape:
        raise ValueError("k and v must share dtype and shape")
    B, Hkv, n_new, d = k.shape
    kp, ks, vp, vs = cache
    cap = kp.shape[2]
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    s = _signs_array(signs)
    rc = _load().oracle_quantize_append_uniform(_ptr(k), _ptr(v), dt, B, Hkv, n_new, d, _ptr(pos),
                                                _ptr(s), bits, _ptr(kp), _ptr(ks), _ptr(vp), _ptr(vs),
                                                cap, threads)
    if rc != 0:
        raise ValueError(f"oracle_quantize_append_uniform failed ({rc})")


def sdpa_cb_decode(q, cache, ctx_lens, signs, bits: int, levels, attn_scale: float,
                   num_kv_heads: int, threads: int = 1) -> np.ndarray:
    """fp64 attention of q over a codebook cache; returns (B, Hq, d) fp64."""
    q, qdt = _input_array(q)
    B, Hq, d = q.shape
    kp, ks, vp, vs = [np.ascontiguousarray(a) for a in cache]
    cap = kp.shape[2]
    ctx = np.ascontiguousarray(ctx_lens, dtype=np.int32)
    s = _signs_array(signs)
    c = _levels_array(levels, bits)
    out = np.empty((B, Hq, d), dtype=np.float64)
    rc = _load().oracle_sdpa_cb_decode(_ptr(q), qdt, B, Hq, num_kv_heads, d, bits, _ptr(c), _ptr(kp),
                                       _ptr(ks), _ptr(vp), _ptr(vs), cap, _ptr(ctx), _ptr(s),
                                       float(attn_scale), _ptr(out), threads)
    if rc != 0:
        raise ValueError(f"oracle_sdpa_cb_decode failed ({rc})")
    return out
