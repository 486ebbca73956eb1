"""CPU pins of the fifth-generation tensor-core encodings the sm_100a kernels
hand-pack (tc.cuh idesc_bf16 and sdesc, tc_tiles.cuh operand_desc and
kstep_bytes).  Expected values are built here field by field from the PTX ISA
layouts of the kind::f16 instruction descriptor and of the shared-memory
matrix descriptor, and compared with what the library's own header code
computes (a host probe compiled with nvcc; no GPU).  Every (M, N, majorness)
that a kernel source passes to idesc_bf16 is checked, and must be a valid
tcgen05.mma shape."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_delta_rule_gdn2_b200", "csrc")


def _kernel_shapes():
    shapes = set()
    pat = re.compile(r"idesc_bf16\(\s*(\d+)\s*,\s*(\d+)\s*,\s*(true|false)\s*,\s*(true|false)\s*\)")
    for f in sorted(os.listdir(CSRC)):
        if f.endswith(".cu"):
            for m in pat.finditer(open(os.path.join(CSRC, f)).read()):
                shapes.add((int(m.group(1)), int(m.group(2)), m.group(3) == "true", m.group(4) == "true"))
    return sorted(shapes)


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("probe") / "tc_desc_probe")
    try:
        subprocess.check_call(["nvcc", "-std=c++17", "--expt-relaxed-constexpr", "-gencode",
                               "arch=compute_100a,code=sm_100a", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                               os.path.join(ROOT, "tests", "tc_desc_probe.cu"), "-o", exe])
    except (OSError, subprocess.CalledProcessError) as e:  # pragma: no cover
        pytest.skip("nvcc unavailable: %s" % e)
    args = []
    for M, N, a, b in _kernel_shapes():
        args += [str(M), str(N), str(int(a)), str(int(b))]
    out = subprocess.check_output([exe] + args, text=True)
    return [l.split() for l in out.splitlines()]


def expected_idesc(M, N, a_mn, b_mn):
    # kind::f16 instruction descriptor (PTX ISA, tcgen05 instruction descriptor table):
    # bits 0-1 sparsity selector, 2 sparsity, 3 saturate, 4-5 D format (1 = f32),
    # 7-9 A format (1 = bf16), 10-12 B format (1 = bf16), 13/14 negate A/B,
    # 15/16 transpose (MN-major) A/B, 17-22 N >> 3, 24-28 M >> 4
    d = 0
    d |= 1 << 4
    d |= 1 << 7
    d |= 1 << 10
    d |= int(a_mn) << 15
    d |= int(b_mn) << 16
    d |= (N >> 3) << 17
    d |= (M >> 4) << 24
    return d


def expected_sdesc(start, lbo, sbo):
    # shared-memory matrix descriptor: bits 0-13 start >> 4, 16-29 leading
    # byte offset >> 4, 32-45 stride byte offset >> 4, 46-48 the fixed 0b001 of
    # sm_100, 49-51 base offset (0: atoms 1 KB aligned), 52 LBO mode (0),
    # 61-63 swizzle mode (2 = 128-byte swizzle)
    return ((start >> 4) & 0x3FFF) | (((lbo >> 4) & 0x3FFF) << 16) | (((sbo >> 4) & 0x3FFF) << 32) | \
        (1 << 46) | (2 << 61)


def test_kernels_use_valid_mma_shapes():
    shapes = _kernel_shapes()
    assert len(shapes) >= 5
    for M, N, _, _ in shapes:
        assert M in (64, 128)
        assert (M == 64 and N % 8 == 0 and 8 <= N <= 256) or (M == 128 and N % 16 == 0 and 16 <= N <= 256)


def test_instruction_descriptors(probe):
    rows = [r for r in probe if r[0] == "idesc"]
    assert len(rows) == len(_kernel_shapes())
    for _, M, N, a, b, val in rows:
        assert int(val) == expected_idesc(int(M), int(N), a == "1", b == "1"), (M, N, a, b, hex(int(val)))
    # a well-known value: M = N = 128, bf16 x bf16 -> f32, both K-major
    assert expected_idesc(128, 128, False, False) == 0x08200490


def test_operand_descriptors(probe):
    seen = 0
    for tag, st, R, s, val, off in (r for r in probe if r[0] in ("kdesc", "mdesc")):
        st, R, s, val, off = int(st), int(R), int(s), int(val), int(off)
        if tag == "kdesc":
            # K-major: 16 bf16 = 32 bytes per k-step inside a 128-byte swizzle
            # row, four per row; then the next 64-column block, R rows of 128 bytes on
            want_off = (s // 4) * R * 128 + (s % 4) * 32
            want = expected_sdesc(st + want_off, 16, 1024)
        else:
            # MN-major: 16 K rows of 128 bytes per k-step; 64-element groups R * 128 bytes apart
            want_off = s * 16 * 128
            want = expected_sdesc(st + want_off, R * 128, 1024)
        assert off == want_off and val == want, (tag, st, R, s)
        # the kernels add off >> 4 to k-step 0's descriptor: no carry out of the start field
        base = expected_sdesc(st, 16 if tag == "kdesc" else R * 128, 1024)
        assert val == base + (off >> 4)
        seen += 1
    assert seen == 2 * 4 * 2 * 8


def test_tf32_rounding_by_integer_add():
    """The WY solve's TF32 operands are rounded by adding 2^12 to the fp32 bit
    pattern (the tensor cores then ignore the low 13 bits).  That is rounding
    of the magnitude to 10 fractional mantissa bits, ties away from zero: checked
    against the rounding computed in fp64 from the value's binary exponent, on
    random values over many binades, on exact ties and at binade edges."""
    import numpy as np
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(200000) * np.exp2(rng.integers(-60, 60, 200000))).astype(np.float32)
    m, e = np.frexp(x.astype(np.float64))  # x = m 2^e, 0.5 <= |m| < 1
    ties = (np.float64(1.0) + (2 * rng.integers(0, 1 << 10, 1000) + 1) * 2.0 ** -11).astype(np.float32)
    edge = np.float32(2.0) - np.float32(2.0 ** -23) * np.arange(1, 600, dtype=np.float32)
    x = np.concatenate([x, ties, -ties, edge, -edge])
    m, e = np.frexp(x.astype(np.float64))
    scaled = np.abs(m) * 2.0 ** 11                       # 11 significant bits kept
    want = np.sign(m) * np.floor(scaled + 0.5) * 2.0 ** (e - 11)
    bits = x.view(np.uint32).astype(np.uint64)
    got = (((bits + 0x1000) & 0xFFFFE000) & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
    assert np.array_equal(got, want)
