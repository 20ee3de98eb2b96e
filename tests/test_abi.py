"""The C-ABI library loads, exports every entry point include/*.h declares,
and rejects invalid arguments on the host before any launch (no GPU needed:
validation fails before the first CUDA call)."""
import ctypes
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent


def declared_symbols():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        text = h.read_text()
        names |= set(re.findall(r"^Q4_API\s+[\w\s\*]+?\b(q4_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from mxfp4_w4a4_block_b200 import build
    build.build()
    import mxfp4_w4a4_block_b200 as q4
    return q4.lib()


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ["q4_amax", "q4_quantize", "q4_dequantize", "q4_sigma_delta_step", "q4_gemm",
              "q4_gemm_workspace_size", "q4_get_device_error", "q4_status_string", "q4_scale_bytes"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(str(ROOT / "mxfp4_w4a4_block_b200" / "libq4.so"))
    for n in declared_symbols():
        assert hasattr(raw, n), n


def test_status_strings_and_version(lib):
    assert lib.q4_version() >= 100
    for s in range(8):
        assert lib.q4_status_string(s)


def test_scale_bytes(lib):
    import mxfp4_w4a4_block_b200 as q4
    assert q4.q4_scale_bytes(q4.NVFP4, 200, 336, q4.LAYOUT_TC) == 256 * 24
    assert q4.q4_scale_bytes(q4.NVFP4, 200, 336, 0) == 200 * 21
    assert q4.q4_scale_bytes(q4.MXFP4, 3, 352, q4.LAYOUT_TC) == 128 * 12
    assert q4.q4_scale_bytes(q4.NVFP4, 10, 17, 0) == 0


def test_workspace_size(lib):
    import mxfp4_w4a4_block_b200 as q4
    assert q4.q4_gemm_workspace_size(q4.NVFP4, 16, 17408, 5120, q4.A_BF16) == 0
    # below one 256-element k-block the activations are quantized once into the workspace
    # (codes 5 x 96 bytes rounded up to 256, then one 128-row band of three 512-byte scale atoms)
    assert q4.q4_gemm_workspace_size(q4.NVFP4, 5, 392, 192, q4.A_BF16) == 512 + 3 * 512
    assert q4.q4_gemm_workspace_size(q4.NVFP4, 8192, 5120, 5120, q4.A_QUANTIZED) == 0
    ws = q4.q4_gemm_workspace_size(q4.NVFP4, 8192, 5120, 5120, q4.A_BF16)
    assert ws == 8192 * 2560 + 8192 * 320


def test_host_validation_without_launch(lib):
    import mxfp4_w4a4_block_b200 as q4
    P = 1 << 20                   # a fake, 16-byte aligned "device" address; never dereferenced
    g = P + 4096
    # block size must match the format
    assert lib.q4_quantize(q4.NVFP4, 32, q4.BF16, P, 4, 64, 64, g, None, P, P, 0, None) == 4
    # NVFP4 needs a tensor scale; MXFP4 must not get one
    assert lib.q4_quantize(q4.NVFP4, 16, q4.BF16, P, 4, 64, 64, None, None, P, P, 0, None) == 1
    assert lib.q4_quantize(q4.MXFP4, 32, q4.BF16, P, 4, 64, 64, g, None, P, P, 0, None) == 1
    # columns must be whole blocks
    assert lib.q4_quantize(q4.NVFP4, 16, q4.BF16, P, 4, 40, 40, g, None, P, P, 0, None) == 3
    # misaligned pointer / row stride
    assert lib.q4_quantize(q4.NVFP4, 16, q4.BF16, P + 2, 4, 64, 64, g, None, P, P, 0, None) == 2
    assert lib.q4_quantize(q4.NVFP4, 16, q4.BF16, P, 4, 64, 68, g, None, P, P, 0, None) == 2
    # Hadamard is MXFP4-only
    assert lib.q4_quantize(q4.NVFP4, 16, q4.BF16, P, 4, 64, 64, g, None, P, P, q4.HADAMARD32, None) == 4
    # empty tensors are a no-op
    assert lib.q4_quantize(q4.NVFP4, 16, q4.BF16, None, 0, 64, 64, g, None, None, None, 0, None) == 0
    # GEMM: K must be a multiple of 64, N of 8
    assert lib.q4_gemm(q4.NVFP4, 16, 4, 8, 96, 0, P, P, g, P, P, g, q4.BF16, P, None, 0, None) == 3
    assert lib.q4_gemm(q4.NVFP4, 16, 4, 12, 64, 0, P, P, g, P, P, g, q4.BF16, P, None, 0, None) == 3
    # GEMM: missing workspace for the quantize-once path
    assert lib.q4_gemm(q4.NVFP4, 16, 4096, 64, 64, q4.A_BF16, P, None, g, P, P, g, q4.BF16, P,
                       None, 0, None) == 7
    # Sigma-Delta: NVFP4 needs s_t
    assert lib.q4_sigma_delta_step(q4.NVFP4, 16, P, 4, 64, P, None, P, P, 0, None) == 1
    # unknown flag bits are rejected; the stall injection is a quantize flag
    assert lib.q4_quantize(q4.NVFP4, 16, q4.BF16, P, 4, 64, 64, g, None, P, P, 1 << 17, None) == 1
    # wait limits outside [1000, 2^40] cycles
    assert lib.q4_set_wait_limit(999) == 1
    assert lib.q4_set_wait_limit((1 << 40) + 1) == 1
    assert lib.q4_set_wait_limit(-5) == 1
    # shared-A GEMM: 1..4 weights, each validated like q4_gemm
    W = q4.Q4GemmWeight
    one = (W * 1)(W(P, P, g, P, 64))
    five = (W * 5)(*[W(P, P, g, P, 64) for _ in range(5)])
    assert lib.q4_gemm_shared_a(q4.NVFP4, 16, 128, 128, P, P, g, one, 0, q4.BF16, None) == 1
    assert lib.q4_gemm_shared_a(q4.NVFP4, 16, 128, 128, P, P, g, five, 5, q4.BF16, None) == 1
    assert lib.q4_gemm_shared_a(q4.NVFP4, 16, 128, 128, P, P, None, one, 1, q4.BF16, None) == 1
    bad_n = (W * 1)(W(P, P, g, P, 12))
    assert lib.q4_gemm_shared_a(q4.NVFP4, 16, 128, 128, P, P, g, bad_n, 1, q4.BF16, None) == 3
    no_gs = (W * 1)(W(P, P, None, P, 64))
    assert lib.q4_gemm_shared_a(q4.NVFP4, 16, 128, 128, P, P, g, no_gs, 1, q4.BF16, None) == 1
    mis = (W * 1)(W(P + 8, P, g, P, 64))
    assert lib.q4_gemm_shared_a(q4.NVFP4, 16, 128, 128, P, P, g, mis, 1, q4.BF16, None) == 2
    assert lib.q4_gemm_shared_a(q4.NVFP4, 16, 128, 96, P, P, g, one, 1, q4.BF16, None) == 3
    # no-alloc GEMM: shape bounds before anything else happens
    assert lib.q4_gemm_a_bf16_noalloc(4, (1 << 31) + 8, 64, P, g, P, P, g, q4.F32, P, None) == 3
    assert lib.q4_gemm_a_bf16_noalloc(4, 16, 96, P, g, P, P, g, q4.F32, P, None) == 3


def test_grouped_host_validation_without_launch(lib):
    """Grouped calls check every entry as the single call would, before any launch."""
    import mxfp4_w4a4_block_b200 as q4
    P = 1 << 20
    g = P + 4096

    def mats(*entries):
        arr = (q4.Q4Matrix * max(len(entries), 1))()
        for i, e in enumerate(entries):
            arr[i] = q4.Q4Matrix(*e)
        return ctypes.addressof(arr), len(entries), arr

    ok = (P, 4, 64, P, g, P, P)
    a, n, keep = mats(ok, ok)
    # more entries than Q4_MAX_GROUP, a negative count, a NULL array
    assert lib.q4_sigma_delta_step_grouped(q4.NVFP4, 16, a, q4.MAX_GROUP + 1, 0, None) == 1
    assert lib.q4_sigma_delta_step_grouped(q4.NVFP4, 16, a, -1, 0, None) == 1
    assert lib.q4_sigma_delta_step_grouped(q4.NVFP4, 16, None, 2, 0, None) == 1
    # nothing to do: no entries, or only empty matrices
    assert lib.q4_sigma_delta_step_grouped(q4.NVFP4, 16, a, 0, 0, None) == 0
    e, n, keep2 = mats((None, 0, 64, None, g, None, None), (None, 5, 0, None, g, None, None))
    assert lib.q4_sr_requant_grouped(q4.NVFP4, 16, e, n, 1, 2, 0, None) == 0
    # one bad entry fails the whole call: missing s_t, ragged columns, misaligned weights,
    # missing residue for the step
    for bad, want in [((P, 4, 64, P, None, P, P), 1), ((P, 4, 40, P, g, P, P), 3),
                      ((P + 4, 4, 64, P, g, P, P), 2), ((P, 4, 64, P, g, None, P), 1)]:
        b, n, keep3 = mats(ok, bad)
        assert lib.q4_sigma_delta_step_grouped(q4.NVFP4, 16, b, n, 0, None) == want
    # MXFP4 entries must not carry s_t; 4/6 scaling is NVFP4-only; codebank visit range
    m, n, keep4 = mats((P, 4, 64, P, g, None, P))
    assert lib.q4_quantize_grouped(q4.MXFP4, 32, q4.F32, m, n, 0, None) == 1
    assert lib.q4_quantize_grouped(q4.MXFP4, 32, q4.F32, m, n, q4.SCALE_46, None) == 4
    assert lib.q4_sigma_delta_codebanks_grouped(q4.NVFP4, 16, a, 2, 0, 0, None) == 1
    # the block size must match the format
    assert lib.q4_sr_requant_grouped(q4.NVFP4, 32, a, 2, 1, 2, 0, None) == 4


def test_grouped_sigma_delta_gemm_validation_without_launch(lib):
    import mxfp4_w4a4_block_b200 as q4
    P = 1 << 20
    g = P + 4096
    arr = (q4.Q4SdGemmEntry * 2)()
    arr[0] = q4.Q4SdGemmEntry(P, P, P, g, P, P, 1024)
    arr[1] = q4.Q4SdGemmEntry(P, P, P, g, P, P, 1020)          # N not a multiple of 8
    a = ctypes.addressof(arr)
    assert lib.q4_sigma_delta_gemm_grouped(q4.NVFP4, 16, 16, 1024, a, 2, q4.BF16, q4.LAYOUT_TC, None) == 3
    assert lib.q4_sigma_delta_gemm_grouped(q4.NVFP4, 16, 16, 1000, a, 1, q4.BF16, q4.LAYOUT_TC, None) == 3
    assert lib.q4_sigma_delta_gemm_grouped(q4.NVFP4, 16, 17, 1024, a, 1, q4.BF16, q4.LAYOUT_TC, None) == 4
    assert lib.q4_sigma_delta_gemm_grouped(q4.MXFP4, 32, 16, 1024, a, 1, q4.BF16, q4.LAYOUT_TC, None) == 4
    assert lib.q4_sigma_delta_gemm_grouped(q4.NVFP4, 16, 16, 1024, a, 1, q4.BF16, 0, None) == 4
    assert lib.q4_sigma_delta_gemm_grouped(q4.NVFP4, 16, 16, 1024, a, q4.MAX_GROUP + 1, q4.BF16,
                                           q4.LAYOUT_TC, None) == 1
    assert lib.q4_sigma_delta_gemm_grouped(q4.NVFP4, 16, 16, 1024, a, 0, q4.BF16, q4.LAYOUT_TC, None) == 0
    arr[0] = q4.Q4SdGemmEntry(P, P, P, None, P, P, 1024)         # missing s_t
    assert lib.q4_sigma_delta_gemm_grouped(q4.NVFP4, 16, 16, 1024, a, 1, q4.BF16, q4.LAYOUT_TC, None) == 1
