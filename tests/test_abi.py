"""The C-ABI library loads and exports every symbol the header declares, and
rejects invalid arguments on the host (no GPU is touched by these tests:
every call here fails validation before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MSA_EXPORT\s+[\w\s\*]*?\b(msa_\w+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_symbols()
    for want in ("msa_index_block_scores", "msa_topk_blocks", "msa_sparse_attn_fwd", "msa_forward",
                 "msa_workspace_size", "msa_status_string", "msa_get_device_error",
                 "msa_kernel_launches", "msa_selftest_wait_timeout", "msa_forward_host",
                 "msa_sparse_attn_fwd_mass", "msa_forward_mass", "msa_decode_paged"):
        assert want in names


def test_library_exports_every_declared_symbol():
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import binding
    lib = ctypes.CDLL(binding.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared in msa.h but not exported"
    assert set(declared_symbols()) == set(msa.EXPORTS)


def _p(**kw):
    import torch
    from block_sparse_long_03_b200 import make_params
    base = dict(B=1, T=256, S=256, Hq=8, Hkv=2, d=128, d_idx=64, block=128, topk=2,
                dtype=torch.bfloat16)
    base.update(kw)
    return make_params(**base)


def test_status_strings():
    from block_sparse_long_03_b200 import binding
    for code, name in binding.STATUS_NAMES.items():
        assert binding.status_string(code).startswith(name)
    assert "unknown" in binding.status_string(99)


def test_workspace_sizes():
    from block_sparse_long_03_b200 import binding
    p = _p()
    ws_attn = binding.msa_workspace_size(p, binding.MSA_WS_SPARSE_ATTN)
    ws_fwd = binding.msa_workspace_size(p, binding.MSA_WS_FORWARD)
    assert ws_attn >= 256 and ws_fwd >= 256
    # forward holds at least the block scores and the ids
    assert ws_fwd >= 256 + 4 * (1 * 256 * 2 * 2) + 4 * (1 * 256 * 2 * 2)
    assert binding.msa_workspace_size(_p(T=0), binding.MSA_WS_FORWARD) == 0
    assert binding.msa_workspace_size(p, 7) == 0
    # the host-buffer call's device buffer holds the forward scratch plus a
    # device copy of every input and output
    ws_host = binding.msa_workspace_size(p, binding.MSA_WS_FORWARD_HOST)
    tensors = 2 * (256 * 2 * 64 + 256 * 64 + 2 * 256 * 8 * 128 + 2 * 256 * 2 * 128) + 4 * 256 * 8
    assert ws_host >= ws_fwd + tensors
    assert binding.msa_workspace_size(_p(T=0), binding.MSA_WS_FORWARD_HOST) == 0


BAD_SHAPES = [
    (dict(T=0), 1), (dict(T=512), 1), (dict(Hq=6, Hkv=4), 1), (dict(topk=0), 1),
    (dict(B=-1), 1), (dict(S=320), 2), (dict(d=96), 2), (dict(block=32), 2),
    (dict(d_idx=24), 2), (dict(Hq=64, Hkv=2), 2), (dict(topk=1000), 2),
    (dict(Hq=512, Hkv=512), 2),
]


@pytest.mark.parametrize("kw,status", BAD_SHAPES)
def test_bad_shapes_rejected_on_host(kw, status):
    from block_sparse_long_03_b200 import binding
    p = _p(**kw)
    fake = ctypes.c_void_p(0x10000)       # never dereferenced: validation fails first
    ws = ctypes.c_void_p(0x20000)
    lib = binding.lib
    assert lib.msa_index_block_scores(ctypes.byref(p), fake, fake, fake, None) == status
    assert lib.msa_topk_blocks(ctypes.byref(p), fake, fake, None) == status
    assert lib.msa_sparse_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, ws,
                                   1 << 30, None) == status
    assert lib.msa_forward(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, ws,
                           1 << 30, None) == status
    assert lib.msa_forward_host(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake,
                                ws, 1 << 30, None) == status
    assert lib.msa_sparse_attn_fwd_mass(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake,
                                        ws, 1 << 30, None) == status
    assert lib.msa_forward_mass(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake,
                                fake, ws, 1 << 30, None) == status


def test_null_and_misaligned_pointers_rejected():
    from block_sparse_long_03_b200 import binding
    lib = binding.lib
    p = _p()
    ok = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)        # 8-byte aligned only
    ws = ctypes.c_void_p(0x20000)
    assert lib.msa_index_block_scores(None, ok, ok, ok, None) == 1
    assert lib.msa_index_block_scores(ctypes.byref(p), None, ok, ok, None) == 1
    assert lib.msa_index_block_scores(ctypes.byref(p), odd, ok, ok, None) == 1
    assert lib.msa_topk_blocks(ctypes.byref(p), ok, None, None) == 1
    assert lib.msa_sparse_attn_fwd(ctypes.byref(p), ok, ok, ok, ok, ok, odd, ws, 1 << 30,
                                   None) == 1
    # workspace: null, misaligned, too small
    assert lib.msa_sparse_attn_fwd(ctypes.byref(p), ok, ok, ok, ok, ok, ok, None, 1 << 30,
                                   None) == 5
    assert lib.msa_sparse_attn_fwd(ctypes.byref(p), ok, ok, ok, ok, ok, ok,
                                   ctypes.c_void_p(0x20010), 1 << 30, None) == 5
    assert lib.msa_forward(ctypes.byref(p), ok, ok, ok, ok, ok, None, ok, ok, ws, 16, None) == 5
    # msa_forward_host checks its device buffer before looking at the host ones
    need = binding.msa_workspace_size(p, binding.MSA_WS_FORWARD_HOST)
    assert lib.msa_forward_host(ctypes.byref(p), ok, ok, ok, ok, ok, None, ok, ok, None, need,
                                None) == 5
    assert lib.msa_forward_host(ctypes.byref(p), ok, ok, ok, ok, ok, None, ok, ok, ws, need - 1,
                                None) == 5
    assert lib.msa_forward_host(ctypes.byref(p), None, ok, ok, ok, ok, None, ok, ok, ws, need,
                                None) == 1
    assert lib.msa_get_device_error(None, None) == 5
    # the mass output must be 16-byte aligned; the workspace rules are the base calls'
    assert lib.msa_sparse_attn_fwd_mass(ctypes.byref(p), ok, ok, ok, ok, ok, ok, odd, ws,
                                        1 << 30, None) == 1
    assert lib.msa_forward_mass(ctypes.byref(p), ok, ok, ok, ok, ok, None, ok, ok, odd, ws,
                                1 << 30, None) == 1
    assert lib.msa_forward_mass(ctypes.byref(p), ok, ok, ok, ok, ok, None, ok, ok, ok, ws, 16,
                                None) == 5


def test_missing_library_fails_loudly(tmp_path):
    """Without libmsa.so the package refuses to import: there is no other
    implementation to fall back to."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "block_sparse_long_03_b200")
    dst = tmp_path / "block_sparse_long_03_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "*.so.*", "csrc",
                                                            "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import block_sparse_long_03_b200"],
                       cwd=str(tmp_path), capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libmsa.so" in r.stderr


def test_decode_paged_rejected_on_host():
    """msa_decode_paged validates its page arguments, shapes and workspace on
    the host before anything is enqueued (no pointer is dereferenced)."""
    import torch
    from block_sparse_long_03_b200 import binding
    lib = binding.lib
    fake = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x20000)

    def call(p, page_size=64, max_pages=64, num_pages=100, ws_bytes=1 << 30, lens=fake):
        return lib.msa_decode_paged(ctypes.byref(p), lens, fake, page_size, max_pages, num_pages,
                                    fake, fake, fake, fake, fake, None, fake, fake, ws, ws_bytes,
                                    None)

    p = _p(B=4, T=1, S=4096, Hq=32, Hkv=8, block=64, topk=8)
    need = binding.msa_workspace_size(p, binding.MSA_WS_DECODE_PAGED)
    assert need > 256
    assert call(p, page_size=0) == 1
    assert call(p, page_size=64, max_pages=63) == 1          # 63 * 64 < S
    assert call(p, num_pages=0) == 1
    assert call(p, lens=None) == 1
    assert call(p, lens=ctypes.c_void_p(0x10004)) == 1       # misaligned
    assert call(p, ws_bytes=need - 1) == 5
    p32 = _p(B=4, T=1, S=4096, Hq=32, Hkv=8, block=64, topk=8, dtype=torch.float32)
    assert call(p32) == 2
    assert binding.msa_workspace_size(p32, binding.MSA_WS_DECODE_PAGED) == 0
    wide = _p(B=4, T=8, S=4096, Hq=32, Hkv=8, block=64, topk=8)   # T * G = 64 > 32
    assert call(wide) == 2
    assert call(_p(T=0)) == 1


def test_bf16_without_tensor_core_path_is_unsupported():
    """A bf16 group size with no tensor-core path (R = 3) is rejected on the
    host instead of running on CUDA cores; fp32 of the same shape is served."""
    import torch
    from block_sparse_long_03_b200 import binding
    lib = binding.lib
    fake = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x20000)
    p = _p(Hq=6, Hkv=2)
    assert binding.msa_workspace_size(p, binding.MSA_WS_SPARSE_ATTN) == 0
    assert binding.msa_workspace_size(p, binding.MSA_WS_FORWARD) == 0
    assert lib.msa_sparse_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, ws,
                                   1 << 30, None) == 2
    assert lib.msa_forward(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, ws,
                           1 << 30, None) == 2
    p32 = _p(Hq=6, Hkv=2, dtype=torch.float32)
    assert binding.msa_workspace_size(p32, binding.MSA_WS_FORWARD) > 0


def test_profile_hook_without_launches():
    """msa_profile_begin/end with nothing launched in between return zero
    totals (no device is touched), and end without begin is harmless."""
    from block_sparse_long_03_b200 import binding
    binding.msa_profile_begin()
    r = binding.msa_profile_end()
    assert r == {"attn_ms": 0.0, "attn_launches": 0, "merge_ms": 0.0, "merge_launches": 0}
    assert binding.msa_profile_end()["attn_launches"] == 0


def test_package_names_resolve():
    """Every name the package exports resolves to the binding (the library
    loads without a device)."""
    import block_sparse_long_03_b200 as msa
    for name in msa.__all__:
        assert getattr(msa, name) is not None, name
