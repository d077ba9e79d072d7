"""The C ABI library without a GPU: it loads, exports every function the
header declares, and rejects bad arguments on the host before touching a
device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("bin_pack", "bin_linear_w1a16", "bitlinear_w1a8", "bitlinear_w1a8_debug",
              "bl_workspace_bytes", "bl_status_string", "bl_device_error", "bl_abi_version"):
        assert n in names, names


def test_library_exports_every_declared_symbol():
    import bit_linear_layers_b200 as bl
    raw = ctypes.CDLL(bl.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), f"{name} declared in bitlinear.h but not exported"
    assert set(declared_functions()) == set(bl.SIGNATURES), "binding and header disagree"


def test_abi_version_and_status_strings():
    import bit_linear_layers_b200 as bl
    assert bl.lib.bl_abi_version() == 1
    for code in (0, -1, -2, -3, -4, -5):
        s = bl.status_string(code)
        assert s and s != "unknown status"
    assert bl.status_string(12345) == "unknown status"


def test_workspace_sizes():
    import bit_linear_layers_b200 as bl
    assert bl.workspace_bytes(bl.BL_OP_PACK_FBI, 0, 4096, 4096) == 0
    assert bl.workspace_bytes(bl.BL_OP_W1A16, 16, 4096, 4096) == 0
    assert bl.workspace_bytes(bl.BL_OP_PACK_BITNET, 0, 4096, 4096) >= 4096 * 16 + 16
    ws = bl.workspace_bytes(bl.BL_OP_W1A8, 512, 5632, 2048)
    assert ws >= 512 * 2048 + 512 * 8 and ws % 256 == 0
    assert bl.workspace_bytes(bl.BL_OP_W1A8, -1, 1, 128) == 0
    ex = bl.workspace_bytes(bl.BL_OP_W1A8_EX, 512, 5632, 2048)
    assert ex >= ws + 512 * 32 + 16 and ex % 256 == 0


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every case below fails validation
ODD = ctypes.c_void_p(0x10001)


@pytest.mark.parametrize("M,N,K,code", [
    (1, 64, 100, -2),      # K not a multiple of 128
    (1, 64, 0, -1),        # K < 1
    (-1, 64, 128, -1),     # negative M
    (1, 0, 128, -1),       # N < 1
    (1 << 31, 1, 128, -2),  # M beyond int32
])
def test_w1a16_shape_validation(M, N, K, code):
    import bit_linear_layers_b200 as bl
    assert bl.lib.bin_linear_w1a16(FAKE, FAKE, FAKE, FAKE, M, N, K, None) == code


def test_null_and_misaligned_pointers_rejected():
    import bit_linear_layers_b200 as bl
    assert bl.lib.bin_linear_w1a16(None, FAKE, FAKE, FAKE, 1, 128, 128, None) == -1
    assert bl.lib.bin_linear_w1a16(ODD, FAKE, FAKE, FAKE, 1, 128, 128, None) == -1
    assert bl.lib.bitlinear_w1a8(FAKE, FAKE, None, FAKE, 1, 128, 128, FAKE, 1 << 20, None) == -1
    # workspace too small
    assert bl.lib.bitlinear_w1a8(FAKE, FAKE, FAKE, FAKE, 4, 128, 128, FAKE, 16, None) == -1
    # unknown quantiser flag; a per-tensor quantiser given the per-token workspace
    assert bl.lib.bitlinear_w1a8_ex(FAKE, FAKE, FAKE, FAKE, 4, 128, 128, 8, FAKE, 1 << 20,
                                    None, None, None, None) == -1
    small = bl.workspace_bytes(bl.BL_OP_W1A8, 4, 128, 128)
    assert bl.lib.bitlinear_w1a8_ex(FAKE, FAKE, FAKE, FAKE, 4, 128, 128, bl.BL_W1A8_NONNEG, FAKE, small,
                                    None, None, None, None) == -1
    assert bl.lib.bin_pack(FAKE, 128, 128, 7, FAKE, FAKE, FAKE, None, 0, None) == -1
    assert bl.lib.bin_pack(FAKE, 128, 128, bl.BL_PACK_BITNET, FAKE, FAKE, FAKE, None, 0, None) == -1
    assert bl.lib.bin_pack(FAKE, 128, 96, bl.BL_PACK_FBI, FAKE, FAKE, None, None, 0, None) == -2


def test_stack_validation_without_device_work():
    import bit_linear_layers_b200 as bl
    N, K = 256, 4096
    Y0, Y1, X = 0x100000, 0x200000, 0x300000  # never dereferenced: every check below is on the host
    job = bl.StackJob(FAKE.value, FAKE.value, Y0, N)
    ws = bl.workspace_bytes(bl.BL_OP_W1A16_STACK, 0, N, 0)
    assert ws >= 256 + 4 * N

    def call(K, first=0, num=1, n_levels=1, ws_bytes=ws, x=X):
        lv = bl.StackLevel(x, K, first, num)
        return bl.lib.bin_linear_w1a16_stack(ctypes.byref(lv), n_levels, ctypes.byref(job), 1, FAKE, ws_bytes, None)

    assert call(4096, n_levels=0) == 0              # empty stack: nothing to do
    assert call(4000) == -2 and call(12544) == -2   # K % 256, more than 48 words per slice
    assert call(4096, first=1) == -1 and call(4096, num=0) == -1
    assert call(4096, ws_bytes=8) == -1
    assert call(4096, x=ODD.value) == -1
    assert call(4096, x=Y0) == -1                   # reads the output of its own level
    assert call(4096, x=Y0 + 2 * N - 2) == -1       # overlaps it
    assert call(4096) == bl.BL_ERR_NO_DEVICE        # valid: stops only at the device

    def stack(specs, jobs, ws_bytes=1 << 20):
        """specs: (x, K, first, num) per level; jobs: (y, N)."""
        lvs = (bl.StackLevel * len(specs))(*[bl.StackLevel(*sp) for sp in specs])
        jbs = (bl.StackJob * len(jobs))(*[bl.StackJob(FAKE.value, FAKE.value, y, n) for y, n in jobs])
        return bl.lib.bin_linear_w1a16_stack(lvs, len(specs), jbs, len(jobs), FAKE, ws_bytes, None)

    # level 1 reads level 0's output exactly: valid
    assert stack([(X, K, 0, 1), (Y0, K, 1, 1)], [(Y0, K), (Y1, 128)]) == bl.BL_ERR_NO_DEVICE
    # ... but not with a different length, nor part of it
    assert stack([(X, K, 0, 1), (Y0, 2048, 1, 1)], [(Y0, K), (Y1, 128)]) == -1
    assert stack([(X, K, 0, 1), (Y0 + 256, K, 1, 1)], [(Y0, 2 * K), (Y1, 128)]) == -1
    # an input written by a later level
    assert stack([(Y1, K, 0, 1), (X, K, 1, 1)], [(Y0, K), (Y1, K)]) == -1
    # two linears writing overlapping outputs
    assert stack([(X, K, 0, 2)], [(Y0, K), (Y0 + 2 * K - 2, K)]) == -1
    assert stack([(X, K, 0, 1), (Y0, K, 1, 1)], [(Y0, K), (Y0, K)]) == -1
    # a linear listed by two levels
    assert stack([(X, K, 0, 1), (Y0, K, 0, 1)], [(Y0, K)]) == -1
    # the workspace must hold a tagged word per output
    assert stack([(X, K, 0, 1), (Y0, K, 1, 1)], [(Y0, K), (Y1, 128)], ws_bytes=256 + 4 * K) == -1


def test_backward_validation_without_device_work():
    import bit_linear_layers_b200 as bl
    ws = bl.workspace_bytes(bl.BL_OP_W1A16_BACKWARD, 64, 256, 256)
    # g = [hi | lo] (64 x 512 bf16), S^T twice, K scales, x^T and dy^T with M padded to 64
    assert ws >= 64 * 256 * 4 + 256 * 256 // 4 + 256 * 4 + 256 * 64 * 2 + 256 * 64 * 2

    def call(M, N, K, dw=FAKE, dalpha=FAKE, ws_bytes=1 << 30, x=FAKE):
        return bl.lib.bin_linear_w1a16_backward(x, FAKE, FAKE, FAKE, FAKE, dw, dalpha, M, N, K, FAKE, ws_bytes, None)

    assert call(4, 192, 256) == -2          # N % 128 != 0
    assert call(4, 256, 200) == -2          # K % 128 != 0
    assert call(4, 256, 256, dalpha=None) == -1  # dW and dalpha come together
    assert call(4, 256, 256, ws_bytes=16) == -1
    assert call(4, 256, 256, x=ODD) == -1


def test_zero_tokens_is_a_noop():
    import bit_linear_layers_b200 as bl
    assert bl.lib.bin_linear_w1a16(None, FAKE, FAKE, None, 0, 128, 128, None) == 0
    assert bl.lib.bitlinear_w1a8(None, FAKE, FAKE, FAKE, 0, 128, 128, None, 0, None) == 0


def test_product_path_has_no_oracle_dependency():
    """The CUDA binding and sources never reference the oracle."""
    pkg = os.path.join(ROOT, "bit_linear_layers_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "liboracle" not in text and "oracle.c" not in text, f
