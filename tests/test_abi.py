"""The C-ABI library: builds for sm_100a, loads, exports every entry point declared in
include/moe.h, and rejects bad arguments on the host before touching the GPU (CPU only)."""
import ctypes as C
import os
import re

import pytest

from tests_support import ROOT
import quantized_moe_router_b200 as qm
from quantized_moe_router_b200 import build as qbuild

HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    if qbuild.stale():
        qbuild.build()
    return qm.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("moe_route_topk", "moe_expert_forward_decode", "moe_expert_forward_prefill", "moe_pack_layer"):
        assert n in names
    assert set(names) == set(qm.SIGNATURES), set(names) ^ set(qm.SIGNATURES)


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    assert L.moe_abi_version() == 1
    names = [qm.status_name(s) for s in range(6)]
    assert names == ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_CUDA", "MOE_ERR_TIMEOUT",
                     "MOE_ERR_DEVICE_CHECK"]


def test_packed_layer_bytes(L):
    # 4-bit tile = 512 B codes + 64 B scale/zero; an expert has 3*I*H/1024 tiles; experts are
    # 256-byte aligned after a 32-byte header and 16 bytes per expert entry.
    E, H, I = 256, 2048, 512
    per_expert = 3 * I * H // 1024 * 576
    assert per_expert == 1769472  # = the canonical bytes: I*H*3/2 codes + 4 bytes per group
    head = (32 + 16 * E + 255) // 256 * 256
    assert qm.packed_layer_bytes(E, H, I, [4] * E) == head + E * per_expert
    mixed = [4, 6, 8]
    per = {4: 576, 6: 832, 8: 1088}
    want = (32 + 16 * 3 + 255) // 256 * 256
    for b in mixed:
        want += (3 * 64 * 128 // 1024 * per[b] + 255) // 256 * 256
    assert qm.packed_layer_bytes(3, 128, 64, mixed) == want
    arr = (C.c_int32 * 2)(4, 5)
    assert L.moe_packed_layer_bytes(2, 128, 64, C.cast(arr, C.c_void_p)) == 0
    arr = (C.c_int32 * 1)(4)
    assert L.moe_packed_layer_bytes(1, 100, 64, C.cast(arr, C.c_void_p)) == 0


def test_workspace_bytes_validation(L):
    assert L.moe_workspace_bytes(1, 2048, 512, 256, 8, 0) > 0
    assert L.moe_workspace_bytes(4096, 2048, 512, 256, 8, 1) > L.moe_workspace_bytes(1, 2048, 512, 256, 8, 1)
    for bad in [(0, 2048, 512, 256, 8, 0), (1, 2000, 512, 256, 8, 0), (1, 2048, 500, 256, 8, 0),
                (1, 2048, 512, 256, 0, 0), (1, 2048, 512, 4, 8, 0), (1, 2048, 512, 2048, 8, 0),
                (1, 2048, 512, 256, 33, 0), (1, 2048, 512, 256, 8, 7)]:
        assert L.moe_workspace_bytes(*bad) == 0, bad


def test_host_validation_before_any_launch(L):
    fake = 1 << 20  # aligned non-null address; never dereferenced because validation fails first
    ws_small = 16
    rc = L.moe_expert_forward_decode(fake, fake, None, fake, 1, 2048, 512, 256, 8, fake, None, None, fake, ws_small, None)
    assert rc == qm.MOE_ERR_INVALID_ARG
    rc = L.moe_expert_forward_prefill(fake, fake, None, fake, 4, 2048, 512, 256, 8, fake, None, None, fake, ws_small, None)
    assert rc == qm.MOE_ERR_INVALID_ARG
    rc = L.moe_expert_forward_decode(None, fake, None, fake, 1, 2048, 512, 256, 8, fake, None, None, fake, 1 << 30, None)
    assert rc == qm.MOE_ERR_INVALID_ARG
    rc = L.moe_expert_forward_decode(fake + 2, fake, None, fake, 1, 2048, 512, 256, 8, fake, None, None, fake, 1 << 30, None)
    assert rc == qm.MOE_ERR_INVALID_ARG  # x not 16-byte aligned
    rc = L.moe_expert_forward_decode(fake, fake, None, fake + 16, 1, 2048, 512, 256, 8, fake, None, None, fake, 1 << 30, None)
    assert rc == qm.MOE_ERR_INVALID_ARG  # packed layer not 256-byte aligned
    assert L.moe_route_topk(fake, fake, None, 1, 100, 8, 2, fake, fake, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(fake, fake, None, 1, 128, 8, 9, fake, fake, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(fake, None, None, 1, 128, 8, 2, fake, fake, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_pack_layer(None, 1, 128, 64, fake, 1 << 20, None) == qm.MOE_ERR_INVALID_ARG
    src = (qm.ExpertSrc * 1)()
    src[0].bits = 5
    assert L.moe_pack_layer(C.cast(src, C.c_void_p), 1, 128, 64, fake, 1 << 20, None) == qm.MOE_ERR_INVALID_ARG
    # the two halves of prefill: workspace too small, null or misaligned pointers, bad shape
    big = 1 << 30
    assert L.moe_prefill_route(fake, fake, None, 4, 2048, 512, 256, 8, None, None, fake, ws_small, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_prefill_route(fake, None, None, 4, 2048, 512, 256, 8, None, None, fake, big, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_prefill_route(fake + 2, fake, None, 4, 2048, 512, 256, 8, None, None, fake, big, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_prefill_route(fake, fake, None, 4, 2048, 512, 256, 33, None, None, fake, big, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_prefill_experts(fake, fake, 4, 2048, 512, 256, 8, fake, fake, ws_small, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_prefill_experts(fake, None, 4, 2048, 512, 256, 8, fake, fake, big, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_prefill_experts(fake, fake, 4, 2048, 512, 256, 8, fake + 8, fake, big, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_prefill_experts(fake, fake, 4, 2000, 512, 256, 8, fake, fake, big, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_workspace_init(None, 1024, None) == qm.MOE_ERR_INVALID_ARG
    assert L.moe_get_device_status(None, None) == qm.MOE_ERR_INVALID_ARG
    # the allocation-free decode call checks its arguments on the host as the workspace call
    # does, before it touches the device (so these hold without a GPU as well)
    nf = L.moe_expert_forward_decode_noalloc
    assert nf(None, fake, None, fake, 1, 2048, 512, 256, 8, fake, None, None, None) == qm.MOE_ERR_INVALID_ARG
    assert nf(fake + 2, fake, None, fake, 1, 2048, 512, 256, 8, fake, None, None, None) == qm.MOE_ERR_INVALID_ARG
    assert nf(fake, fake, None, fake + 16, 1, 2048, 512, 256, 8, fake, None, None, None) == qm.MOE_ERR_INVALID_ARG
    assert nf(fake, fake, None, fake, 1, 100, 512, 256, 8, fake, None, None, None) == qm.MOE_ERR_INVALID_ARG
    assert nf(fake, fake, None, fake, 33, 2048, 512, 256, 8, fake, None, None, None) == qm.MOE_ERR_UNSUPPORTED
    assert nf(fake, fake, None, fake, 1, 16384, 512, 256, 8, fake, None, None, None) == qm.MOE_ERR_UNSUPPORTED
    assert L.moe_expert_forward_decode(fake, fake, None, fake, 33, 2048, 512, 256, 8, fake, None, None, fake, 1 << 30,
                                       None) in (qm.MOE_ERR_UNSUPPORTED, qm.MOE_ERR_CUDA)


def test_quantizer_host_validation(L):
    fake = 1 << 20
    P = qm.HqqParams

    def q(w=fake, rows=4, cols=128, bits=4, prm=None, codes=fake, s=fake, z=fake, it=None):
        pp = None if prm is None else C.addressof(prm)
        return L.moe_quantize_hqq(w, rows, cols, bits, pp, codes, s, z, it, None)

    assert q(rows=0) == qm.MOE_OK                 # nothing to do: nothing launched
    assert q(cols=100) == qm.MOE_ERR_INVALID_ARG
    assert q(cols=0) == qm.MOE_ERR_INVALID_ARG
    assert q(rows=-1) == qm.MOE_ERR_INVALID_ARG
    assert q(bits=5) == qm.MOE_ERR_INVALID_ARG
    assert q(w=None) == qm.MOE_ERR_INVALID_ARG
    assert q(codes=None) == qm.MOE_ERR_INVALID_ARG
    assert q(s=None) == qm.MOE_ERR_INVALID_ARG
    assert q(w=fake + 8) == qm.MOE_ERR_INVALID_ARG       # w not 16-byte aligned
    assert q(codes=fake + 2) == qm.MOE_ERR_INVALID_ARG
    assert q(z=fake + 1) == qm.MOE_ERR_INVALID_ARG
    assert q(it=fake + 2) == qm.MOE_ERR_INVALID_ARG
    for bad in (P(0.0, 10.0, 1.01, 20), P(1.5, 10.0, 1.01, 20), P(0.7, 0.0, 1.01, 20),
                P(0.7, float("inf"), 1.01, 20), P(0.7, 10.0, 0.9, 20), P(0.7, 10.0, float("nan"), 20),
                P(0.7, 10.0, 1.01, -1), P(0.7, 10.0, 1.01, 1001)):
        assert q(prm=bad) == qm.MOE_ERR_INVALID_ARG, (bad.lp_norm, bad.beta, bad.kappa, bad.iters)
    assert q(rows=0, prm=P(0.7, 10.0, 1.01, 2000)) == qm.MOE_ERR_INVALID_ARG   # params checked first


def test_binding_refuses_tensors_the_library_cannot_take(L):
    """The C ABI takes raw device pointers; the binding refuses host tensors, wrong dtypes,
    wrong shapes and strided views before anything reaches the library (CPU only)."""
    import torch
    T, H, E, I, k = 2, 128, 4, 64, 2
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    wr = torch.zeros((E, H), dtype=torch.float32)
    packed = torch.zeros(1 << 16, dtype=torch.uint8)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.forward_decode(x, wr, None, packed, I, E, k, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.forward_prefill(x, wr, None, packed, I, E, k, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.route_topk(x, wr, None, k)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.prefill_route(x, wr, None, I, E, k, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.prefill_experts(x, packed, I, E, k, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.forward_decode_noalloc(x, wr, None, packed, I, E, k)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.quantize_hqq(torch.zeros((4, 128), dtype=torch.bfloat16), 4)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.device_status(ws)
    ex = {"bits": 4, "codes": [torch.zeros((I, H // 2), dtype=torch.uint8)] * 2 + [torch.zeros((H, I // 2), dtype=torch.uint8)],
          "scale": [torch.zeros((I, H // 64), dtype=torch.float16)] * 2 + [torch.zeros((H, I // 64), dtype=torch.float16)],
          "zero": [torch.zeros((I, H // 64), dtype=torch.float16)] * 2 + [torch.zeros((H, I // 64), dtype=torch.float16)]}
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm.pack_layer([ex], H, I)
    # dtype, shape and layout checks come from the same helper
    with pytest.raises(ValueError, match="2-D"):
        qm.quantize_hqq(torch.zeros(128, dtype=torch.bfloat16), 4)
    with pytest.raises(ValueError, match="2-D"):
        qm.forward_decode(torch.zeros(H, dtype=torch.bfloat16), wr, None, packed, I, E, k, ws)


def test_tensor_check_helper():
    import torch
    qm._dev(None, "bias", torch.float32, optional=True)
    with pytest.raises(ValueError, match="required"):
        qm._dev(None, "x", torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm._dev(torch.zeros(3), "x", torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qm._dev(object(), "x", torch.float32)


def test_header_is_plain_c_and_links(tmp_path, L):
    """A C11 translation unit can include include/moe.h and take every entry point's address, and
    links against the library (the ABI is C, not C++)."""
    import subprocess
    names = declared_functions()
    src = tmp_path / "abi_check.c"
    body = "\n".join(f"    p[{i}] = (void (*)(void)){n};" for i, n in enumerate(names))
    src.write_text('#include "moe.h"\n#include <stdio.h>\n\nint main(void) {\n'
                   f'    void (*p[{len(names)}])(void);\n{body}\n'
                   f'    for (int i = 0; i < {len(names)}; ++i) if (!p[i]) return 1;\n'
                   '    printf("%s\\n", moe_status_str(MOE_OK));\n    return 0;\n}\n')
    libdir = os.path.dirname(qm.LIB_PATH)
    exe = tmp_path / "abi_check"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lmoe_b200", "-Wl,-rpath," + libdir,
                    "-Wl,-rpath,/usr/local/cuda/lib64", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "MOE_OK", out
