"""Expert cache (moe_cache_* of include/moe.h): its host logic on the CPU.

The cache's source (quantized_moe_router_b200/csrc/moe_cache.cu) is host code whose only device
operation is an asynchronous host-to-device copy. Here it is compiled with tests/cache_host_shim.cpp,
which turns that copy into a memcpy into a host buffer standing in for the device pool, so that
whole request/commit sequences run without a GPU. After each commit the test resolves every
requested expert the way the forward kernels do (layer header address + the entry's offset) and
compares the bytes there with the expert's bytes in the host layer.
"""
import ctypes as C
import os
import subprocess

import numpy as np
import pytest

from tests_support import ROOT
import quantized_moe_router_b200 as qm

SRC = os.path.join(ROOT, "quantized_moe_router_b200", "csrc", "moe_cache.cu")
SHIM = os.path.join(ROOT, "tests", "cache_host_shim.cpp")
OK, INVALID, UNSUPPORTED, CUDA = qm.MOE_OK, qm.MOE_ERR_INVALID_ARG, qm.MOE_ERR_UNSUPPORTED, qm.MOE_ERR_CUDA
vp, i32 = C.c_void_p, C.c_int

# packed format (documented with moe_pack_layer): 32-byte header, 16-byte entries, 256-byte aligned
# expert blocks of 16 x 64 tiles of 576 / 832 / 1088 bytes for 4 / 6 / 8-bit codes
MAGIC, VERSION = 0x50454F4D, 2
TILE = {4: 576, 6: 832, 8: 1088}


def align(v, a=256):
    return (v + a - 1) // a * a


def expert_bytes(H, I, b):
    return ((I // 8) * (H // 64) + (H // 16) * (I // 64)) * TILE[b]


def host_layer(rng, E, H, I, widths):
    """A packed layer as moe_pack_layer lays it out, with random expert bytes."""
    start = align(32 + 16 * E)
    offs, o = [], start
    for b in widths:
        offs.append(o)
        o = align(o + expert_bytes(H, I, b))
    buf = rng.integers(0, 256, o, dtype=np.uint8)
    buf[:32] = 0
    buf[:20].view(np.uint32)[:] = [MAGIC, VERSION, E, H, I]
    for e, (off, b) in enumerate(zip(offs, widths)):
        ent = buf[32 + 16 * e: 48 + 16 * e]
        ent[:8].view(np.uint64)[0] = off
        ent[8:16].view(np.int32)[:] = [b, 0]
    return buf, offs


@pytest.fixture(scope="module")
def L(tmp_path_factory):
    out = tmp_path_factory.mktemp("cache") / "libcache_host.so"
    # -Bsymbolic: the library's calls bind to the shim's copy even when the process has loaded the
    # CUDA runtime (torch does) into the global symbol scope
    subprocess.run(["g++", "-std=c++17", "-O1", "-fPIC", "-shared", "-Wl,-Bsymbolic", "-I/usr/local/cuda/include",
                    "-I", os.path.join(ROOT, "include"), "-x", "c++", SRC, "-x", "c++", SHIM, "-o", str(out)],
                   check=True)
    lib = C.CDLL(str(out))
    lib.moe_cache_pool_bytes.restype = C.c_size_t
    lib.moe_cache_pool_bytes.argtypes = [i32, vp, vp, i32]
    lib.moe_cache_create.argtypes = [i32, vp, vp, i32, i32, vp, C.c_size_t, vp]
    lib.moe_cache_destroy.argtypes = [vp]
    lib.moe_cache_request.argtypes = [vp, i32, vp, i32, vp, vp, vp]
    lib.moe_cache_commit.argtypes = [vp, vp, vp]
    lib.moe_cache_slot_of.argtypes = [vp, i32, i32]
    lib.moe_cache_stats.argtypes = [vp, vp, vp, vp]
    lib.shim_fail_after.argtypes = [i32]
    lib.shim_copies.restype = C.c_long
    lib.shim_set_device_status.argtypes = [i32]
    return lib


class Cache:
    """One cache over host layers, with a host buffer as its pool."""

    def __init__(self, L, layers, slots, keep_recent=1, pool_extra=0):
        self.L, self.layers = L, layers
        n = len(layers)
        self.ptrs = (vp * n)(*[a.ctypes.data for a in layers])
        self.sizes = (C.c_size_t * n)(*[a.size for a in layers])
        self.need = L.moe_cache_pool_bytes(n, C.cast(self.ptrs, vp), C.cast(self.sizes, vp), slots)
        assert self.need > 0
        self.raw = np.zeros(self.need + pool_extra + 256, np.uint8)
        self.base = align(self.raw.ctypes.data)
        self.pool = self.raw[self.base - self.raw.ctypes.data:]
        self.h = vp()
        rc = L.moe_cache_create(n, C.cast(self.ptrs, vp), C.cast(self.sizes, vp), slots, keep_recent, self.base,
                                self.need + pool_extra, C.byref(self.h))
        assert rc == OK, rc

    def request(self, layer, experts):
        arr = (C.c_int32 * max(1, len(experts)))(*experts)
        le = (C.c_int32 * max(1, len(experts)))()
        ls = (C.c_int32 * max(1, len(experts)))()
        nl = C.c_int(-1)
        rc = self.L.moe_cache_request(self.h, layer, C.cast(arr, vp), len(experts), C.cast(le, vp), C.cast(ls, vp),
                                      C.byref(nl))
        return rc, list(le[:max(nl.value, 0)]), list(ls[:max(nl.value, 0)])

    def commit(self):
        out = vp()
        rc = self.L.moe_cache_commit(self.h, None, C.byref(out))
        return rc, (out.value or 0) - self.base

    def slot(self, layer, e):
        return self.L.moe_cache_slot_of(self.h, layer, e)

    def stats(self):
        v = [C.c_uint64() for _ in range(3)]
        assert self.L.moe_cache_stats(self.h, *[C.byref(x) for x in v]) == OK
        return tuple(x.value for x in v)

    def resolve(self, hdr_off, e):
        """The bytes a forward kernel reads for expert e through the header at pool offset hdr_off."""
        hdr = self.pool[hdr_off:]
        head = hdr[:20].view(np.uint32)
        E, H, I = int(head[2]), int(head[3]), int(head[4])
        assert (int(head[0]), int(head[1])) == (MAGIC, VERSION)
        ent = hdr[32 + 16 * e: 48 + 16 * e]
        off, b = int(ent[:8].view(np.uint64)[0]), int(ent[8:12].view(np.int32)[0])
        assert off % 256 == 0 and hdr_off + off + expert_bytes(H, I, b) <= self.need, "entry leaves the pool"
        return hdr[off: off + expert_bytes(H, I, b)], b

    def close(self):
        self.L.moe_cache_destroy(self.h)


def host_expert(layer_buf, offs, widths, H, I, e):
    return layer_buf[offs[e]: offs[e] + expert_bytes(H, I, widths[e])]


def test_layer_builder_matches_the_library_sizes():
    for E, H, I, widths in ((6, 128, 64, [4, 6, 8, 4, 6, 8]), (3, 256, 128, [8, 8, 4])):
        buf, _ = host_layer(np.random.default_rng(0), E, H, I, widths)
        assert buf.size == qm.packed_layer_bytes(E, H, I, widths)


def test_pool_bytes_and_create_validation(L):
    rng = np.random.default_rng(1)
    E, H, I = 6, 128, 64
    widths = [4, 6, 8, 4, 4, 6]
    a, _ = host_layer(rng, E, H, I, widths)
    b, _ = host_layer(rng, E, H, I, widths[::-1])
    ptrs = (vp * 2)(a.ctypes.data, b.ctypes.data)
    sizes = (C.c_size_t * 2)(a.size, b.size)
    n = L.moe_cache_pool_bytes(2, C.cast(ptrs, vp), C.cast(sizes, vp), 3)
    assert n == 2 * align(32 + 16 * E) + 3 * align(expert_bytes(H, I, 8))
    assert L.moe_cache_pool_bytes(2, C.cast(ptrs, vp), C.cast(sizes, vp), 0) == 0

    def create(layers, slots=3, keep=1, pool=1 << 20, pool_bytes=None, sizes_=None):
        p = (vp * len(layers))(*[x.ctypes.data for x in layers])
        s = (C.c_size_t * len(layers))(*(sizes_ or [x.size for x in layers]))
        h = vp()
        rc = L.moe_cache_create(len(layers), C.cast(p, vp), C.cast(s, vp), slots, keep, pool,
                                n if pool_bytes is None else pool_bytes, C.byref(h))
        if rc == OK:
            L.moe_cache_destroy(h)
        return rc

    assert create([a, b]) == OK
    bad = a.copy()
    bad[0] ^= 1
    assert create([bad]) == INVALID                        # magic
    c, _ = host_layer(rng, 5, H, I, widths[:5])
    assert create([a, c]) == INVALID                       # E differs between layers
    assert create([a], sizes_=[a.size - 1]) == INVALID     # last expert runs past the buffer
    mis = a.copy()
    mis[32:40].view(np.uint64)[0] += 16
    assert create([mis]) == INVALID                        # expert offset not 256-aligned
    wb = a.copy()
    wb[40:44].view(np.int32)[0] = 5
    assert create([wb]) == INVALID                         # width 5
    assert create([a], slots=0) == INVALID
    assert create([a], keep=0) == INVALID and create([a], keep=9) == INVALID
    assert create([a], pool=(1 << 20) + 16) == INVALID     # pool not 256-aligned
    assert create([a, b], pool_bytes=n - 1) == INVALID     # pool too small
    assert create([a], pool=0) == INVALID


def test_requests_and_commits_resolve_to_the_host_bytes(L):
    rng = np.random.default_rng(2)
    E, H, I = 6, 128, 64
    widths = [[4, 6, 8, 4, 6, 8], [8, 4, 4, 6, 6, 8]]
    built = [host_layer(rng, E, H, I, w) for w in widths]
    cache = Cache(L, [x[0] for x in built], slots=4)
    seq = [(0, [0, 1]), (1, [2, 3, 3]), (0, [1, 4]), (1, [0, 5, 2]), (0, [0, 1, 2, 3]), (1, [5]),
           (0, []), (1, [1, 2, 3, 4])]
    resident = set()
    for layer, want in seq:
        before = {e: cache.slot(layer, e) for e in range(E)}
        rc, loads, slots = cache.request(layer, want)
        assert rc == OK
        assert loads == [e for e in dict.fromkeys(want) if before[e] < 0]
        assert len(set(slots)) == len(slots) and all(0 <= s < 4 for s in slots)
        copies = L.shim_copies()
        rc, hdr = cache.commit()
        assert rc == OK
        assert L.shim_copies() - copies == len(loads) + 1      # the experts, then the header
        buf, offs = built[layer]
        for e in want:
            got, b = cache.resolve(hdr, e)
            assert b == widths[layer][e]
            assert np.array_equal(got, host_expert(buf, offs, widths[layer], H, I, e)), (layer, e)
        resident = {(l, e) for l in range(2) for e in range(E) if cache.slot(l, e) >= 0}
        assert len(resident) <= 4
        assert all((layer, e) in resident for e in want)
    hits, misses, ev = cache.stats()
    assert hits + misses == sum(len(set(w)) for _, w in seq)
    assert misses - ev == len(resident)    # every load either filled a free slot or evicted
    cache.close()


def test_least_recently_requested_expert_is_evicted(L):
    rng = np.random.default_rng(3)
    E, H, I = 8, 128, 64
    buf, _ = host_layer(rng, E, H, I, [4] * E)
    cache = Cache(L, [buf], slots=3)
    assert cache.request(0, [0, 1, 2])[1:] == ([0, 1, 2], [0, 1, 2])   # free slots in order
    assert cache.commit()[0] == OK
    assert cache.request(0, [3])[1:] == ([3], [0])    # all three equally old: lowest slot
    assert cache.commit()[0] == OK
    assert cache.request(0, [1, 4])[1:] == ([4], [2])  # 1 is a hit; 2 is now the oldest
    assert cache.commit()[0] == OK
    assert [cache.slot(0, e) for e in range(6)] == [-1, 1, -1, 0, 2, -1]
    assert cache.request(0, [5, 6])[1:] == ([5, 6], [0, 1])   # 3 (request 2), then 1 (request 3, slot 1 < 2)
    assert cache.commit()[0] == OK
    assert cache.stats() == (1, 7, 4)
    cache.close()


def test_recent_requests_are_protected(L):
    rng = np.random.default_rng(4)
    E, H, I = 8, 128, 64
    buf, _ = host_layer(rng, E, H, I, [6] * E)
    cache = Cache(L, [buf, buf], slots=3, keep_recent=2)
    assert cache.request(0, [0, 1])[0] == OK and cache.commit()[0] == OK
    before = ([cache.slot(l, e) for l in range(2) for e in range(E)], cache.stats())
    # the previous request's experts may still be in use: only one slot is free for two misses
    assert cache.request(1, [2, 3])[0] == UNSUPPORTED
    assert ([cache.slot(l, e) for l in range(2) for e in range(E)], cache.stats()) == before
    assert cache.request(1, [2])[1:] == ([2], [2])
    assert cache.commit()[0] == OK
    # now request 1 is two requests old: its experts may go, request 2's may not
    assert cache.request(0, [5, 6])[1:] == ([5, 6], [0, 1])
    assert cache.commit()[0] == OK
    assert cache.slot(1, 2) == 2
    cache.close()


def test_more_distinct_experts_than_slots_is_refused(L):
    rng = np.random.default_rng(5)
    buf, _ = host_layer(rng, 8, 128, 64, [4] * 8)
    cache = Cache(L, [buf], slots=3)
    assert cache.request(0, [0, 1, 2, 3])[0] == UNSUPPORTED
    assert cache.request(0, [0, 1, 2, 2, 1, 0])[0] == OK     # duplicates count once
    assert cache.stats() == (0, 3, 0)
    cache.close()


def test_uncommitted_request_is_replaced(L):
    rng = np.random.default_rng(6)
    buf, _ = host_layer(rng, 8, 128, 64, [8] * 8)
    cache = Cache(L, [buf], slots=2)
    assert cache.request(0, [0, 1])[0] == OK and cache.commit()[0] == OK
    copies = L.shim_copies()
    assert cache.request(0, [2, 3])[1:] == ([2, 3], [0, 1])      # not committed ...
    assert cache.request(0, [1, 4])[1:] == ([4], [0])             # ... so 0 and 1 are back
    assert L.shim_copies() == copies                              # requests copy nothing
    assert cache.commit()[0] == OK
    assert [cache.slot(0, e) for e in range(5)] == [-1, 1, -1, -1, 0]
    assert cache.stats() == (1, 3, 1)
    cache.close()


def test_failed_commit_leaves_the_experts_absent(L):
    rng = np.random.default_rng(7)
    E, H, I = 8, 128, 64
    widths = [4, 8] * 4
    buf, offs = host_layer(rng, E, H, I, widths)
    cache = Cache(L, [buf], slots=3)
    assert cache.request(0, [0, 1])[0] == OK and cache.commit()[0] == OK
    L.shim_fail_after(1)                 # the second copy of the next commit fails
    try:
        assert cache.request(0, [2, 3, 0])[1:] == ([2, 3], [2, 1])
        assert cache.commit()[0] == CUDA
    finally:
        L.shim_fail_after(-1)
    assert [cache.slot(0, e) for e in range(4)] == [0, -1, -1, -1]   # 1 was evicted, 2 and 3 not loaded
    assert cache.commit()[0] == INVALID                               # nothing pending any more
    L.shim_set_device_status(UNSUPPORTED)
    try:
        assert cache.request(0, [2])[0] == OK
        copies = L.shim_copies()
        assert cache.commit()[0] == UNSUPPORTED
        assert L.shim_copies() == copies and cache.slot(0, 2) == -1
    finally:
        L.shim_set_device_status(OK)
    assert cache.request(0, [2, 3, 0])[0] == OK
    rc, hdr = cache.commit()
    assert rc == OK
    for e in (0, 2, 3):
        assert np.array_equal(cache.resolve(hdr, e)[0], host_expert(buf, offs, widths, H, I, e))
    cache.close()


def test_invalid_calls(L):
    rng = np.random.default_rng(8)
    buf, _ = host_layer(rng, 4, 128, 64, [4] * 4)
    cache = Cache(L, [buf], slots=2)
    assert cache.commit()[0] == INVALID            # no request
    assert cache.request(1, [0])[0] == INVALID     # no layer 1
    assert cache.request(0, [4])[0] == INVALID     # no expert 4
    assert cache.request(0, [-1])[0] == INVALID
    assert cache.slot(0, 9) == -1 and cache.slot(3, 0) == -1
    assert L.moe_cache_stats(None, None, None, None) == INVALID
    assert L.moe_cache_slot_of(None, 0, 0) == -1
    cache.close()
