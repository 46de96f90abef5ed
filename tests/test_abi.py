"""The C-ABI library loads and exports every entry point include/paro.h
declares; host-only calls validate their arguments (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "paro.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(paro_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from rotated_w4_linear_b200 import build, binding
    build.build()
    return binding.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert "paro_rotate" in names and "paro_linear" in names
    for n in names:
        assert hasattr(L, n), n


def test_binding_names_match_header():
    from rotated_w4_linear_b200 import binding
    for n in _declared():
        assert n in binding._SIGS, n


def test_pack_size(L):
    from rotated_w4_linear_b200 import binding
    qb, sb, zb = binding.paro_pack_size(4096, 6144)
    assert qb == 4096 * 6144 // 2
    assert sb == 6144 // 16 * 32 * 8 * 4 and zb == 6144 // 16 * 32 * 8
    assert binding.paro_pack_size(384, 48)[2] == 48 // 16 * 4 * 8       # 3 groups padded to 4
    # 0.5 + 2/128 + 0.5/128 bytes per weight
    assert (qb + sb + zb) / (4096 * 6144) == pytest.approx(0.5 + 2 / 128 + 0.5 / 128)


@pytest.mark.parametrize("inf,outf", [(100, 64), (128, 20), (0, 16), (-128, 16)])
def test_bad_shapes_rejected(L, inf, outf):
    from rotated_w4_linear_b200 import binding
    with pytest.raises(binding.ParoError) as e:
        binding.paro_pack_size(inf, outf)
    assert e.value.status == 1
    assert "must be" in L.paro_last_error().decode()


def test_null_arguments_rejected_before_any_launch(L):
    assert L.paro_rotate(None, None, None, 4, None) == 1
    assert b"rot is null" in L.paro_last_error()
    assert L.paro_linear(None, None, None, None, None, None, 4, 256, 64, None, 0, None) == 1
    b = ctypes.c_size_t()
    assert L.paro_linear_workspace_size(16, 4096, 4096, ctypes.byref(b)) == 0 and b.value > 0
    assert L.paro_rot_create(None, 256, 128, 8, 64, None, None, None) == 1
    assert L.paro_rot_destroy(None) == 0


def test_wait_selftest_limit_checked_before_launch(L):
    assert L.paro_check_wait_timeout(0, None) == 1
    assert L.paro_check_wait_timeout(2000001, None) == 1
    assert b"limit_us" in L.paro_last_error()


def test_unsupported_group(L):
    h = ctypes.c_void_p()
    assert L.paro_rot_create(ctypes.byref(h), 512, 32, 8, 16, None, None, None) == 2
    assert L.paro_rot_create(ctypes.byref(h), 256, 64, 8, 33, None, None, None) == 1      # P > group / 2
    assert L.paro_rot_create(ctypes.byref(h), 384, 256, 8, 64, None, None, None) == 1     # in % 256
    b = ctypes.c_size_t()
    assert L.paro_pack_size_ex(4096, 64, 512, ctypes.byref(b), ctypes.byref(b), ctypes.byref(b)) == 2


def test_pack_size_group_256_is_the_group_128_format(L):
    from rotated_w4_linear_b200 import binding
    assert binding.paro_pack_size(4096, 6144, 256) == binding.paro_pack_size(4096, 6144, 128)


def test_pack_size_group_64(L):
    from rotated_w4_linear_b200 import binding
    qb, sb, zb = binding.paro_pack_size(4096, 6144, 64)
    assert qb == 4096 * 6144 // 2
    assert sb == 6144 // 16 * 64 * 8 * 4 and zb == 6144 // 16 * 64 * 8
    # 0.5 + 2/64 + 0.5/64 bytes per weight
    assert (qb + sb + zb) / (4096 * 6144) == pytest.approx(0.5 + 2 / 64 + 0.5 / 64)


def test_prepared_layer_checks_its_arguments_once_on_the_host(L):
    """ParoLinear refuses host tensors and a rotation prepared for another
    group size or width before anything reaches the device."""
    import torch
    from rotated_w4_linear_b200 import binding
    u8 = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(TypeError):
        binding.ParoLinear(None, u8, u8, u8, 128, 16)

    class FakeRot:                        # a handle-shaped stand-in; never passed to the library
        group, in_features, handle = 64, 256, None
    with pytest.raises(ValueError):
        binding.ParoLinear(FakeRot(), u8, u8, u8, 256, 16, group=128)
    with pytest.raises(ValueError):
        binding.ParoLinear(FakeRot(), u8, u8, u8, 384, 16, group=64)
