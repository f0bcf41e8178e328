"""The tcgen05 descriptor encoders (csrc/ptx.cuh, csrc/ptx_bs.cuh), evaluated on
the host, field by field against the descriptor tables of the PTX ISA (no GPU):

* shared memory matrix descriptor (64 bits): start address >> 4 in bits 0-13,
  leading-dimension byte offset >> 4 in 16-29, stride-dimension byte offset >> 4
  in 32-45, the fixed constant 0b001 in 46-48, base offset in 49-51 (0 here:
  every tile is 1024-byte aligned), leading-dimension stride mode in 52 (0,
  relative), 53-60 zero, swizzle mode in 61-63 (0 none, 2 128-byte, 4 64-byte);
* instruction descriptor of kind::f8f6f4 (32 bits): sparsity 0-2 and saturate 3
  zero, D format in 4-5 (1 = F32), A / B format in 7-9 / 10-12 (0 = E4M3),
  negate 13 / 14 zero, A / B major in 15 / 16 (1 = MN-major), N >> 3 in 17-22,
  bit 23 zero, M >> 4 in 24-28, 29-31 zero;
* instruction descriptor of kind::mxf8f6f4.block_scale: the same, except bits
  4-5 hold the B scale-factor id (there is no D-format field), bit 23 the
  scale type (1 = UE8M0) and bits 29-30 the A scale-factor id.

The layouts the kernels need of them: K-major tiles of 128-byte rows with the
128-byte swizzle, 8-row core-matrix groups 1024 bytes apart; the MN-major
64-byte-swizzled B tile of the pair kernel, 8-K-row groups 512 bytes apart;
the MN-major 128-byte-swizzled B tile of the single-CTA kernel, 8-K-row groups
1024 bytes apart, its two 128-column halves 16 KB apart; the scale-factor copy
source, 32 rows of 16 bytes without swizzle, 8-row core matrices 128 bytes
apart."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "fp8_block_scaled_11_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "descriptors", "print_descriptors.cu")


def field(v, lo, width):
    return (v >> lo) & ((1 << width) - 1)


@pytest.fixture(scope="module")
def values(tmp_path_factory):
    nvcc = os.environ.get("NVCC", "nvcc")
    if shutil.which(nvcc) is None:
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp("desc") / "print_descriptors")
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                    "-I", os.path.join(ROOT, "include"), SRC, "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    rows = {}
    for line in out.splitlines():
        name, *nums = line.split()
        rows.setdefault(name, []).append(tuple(int(x) for x in nums))
    return rows


SMEM_FIELDS = [(0, 14), (16, 14), (32, 14), (46, 3), (49, 3), (52, 1), (53, 8), (61, 3)]


def check_smem(v, addr, lbo, sbo, swizzle):
    assert field(v, 0, 14) == (addr & 0x3FFFF) >> 4
    assert field(v, 16, 14) == lbo >> 4
    assert field(v, 32, 14) == sbo >> 4
    assert field(v, 46, 3) == 0b001
    assert field(v, 49, 3) == 0
    assert field(v, 52, 1) == 0
    assert field(v, 53, 8) == 0
    assert field(v, 61, 3) == swizzle
    # nothing outside the table's fields (bits 14-15 and 30-31 are reserved)
    known = sum(((1 << w) - 1) << lo for lo, w in SMEM_FIELDS)
    assert v & ~known == 0


def test_k_major_128b_swizzle(values):
    rows = values["smem_desc_k_sw128"]
    assert len(rows) == 7
    for addr, v in rows:
        check_smem(v, addr, lbo=16, sbo=1024, swizzle=2)


def test_mn_major_64b_swizzle(values):
    for addr, v in values["smem_desc_mn_sw64"]:
        check_smem(v, addr, lbo=16, sbo=512, swizzle=4)


def test_mn_major_128b_swizzle(values):
    """The single-CTA kernel's MN-major B tile: K rows of 128 bytes (128 N
    elements per swizzle atom), 8-K-row groups 1024 bytes apart (stride byte
    offset), the two 128-column halves 16 KB apart (leading byte offset: in
    the MN-major canonical layouts it is the step between atoms along MN)."""
    rows = values["smem_desc_mn_sw128"]
    assert len(rows) == 7
    for addr, v in rows:
        check_smem(v, addr, lbo=16384, sbo=1024, swizzle=2)


def test_scale_factor_copy_source(values):
    for addr, v in values["smem_desc_cp_rows16"]:
        check_smem(v, addr, lbo=16, sbo=128, swizzle=0)


def test_k_step_within_a_swizzled_row(values):
    """The kernels step K by 32 bytes inside a 128-byte swizzled row by moving
    the start address: the encoded start field advances by 2 per step."""
    rows = dict(values["smem_desc_k_sw128"])
    assert field(rows[32], 0, 14) - field(rows[0], 0, 14) == 2
    assert rows[32] - rows[0] == 2          # no other field moves


def check_idesc_common(v, M, N):
    assert field(v, 0, 4) == 0          # dense, no saturate
    assert field(v, 7, 3) == 0          # A: E4M3
    assert field(v, 10, 3) == 0         # B: E4M3
    assert field(v, 13, 2) == 0         # no negation
    assert field(v, 15, 1) == 0         # A K-major
    assert field(v, 17, 6) == N >> 3
    assert field(v, 24, 5) == M >> 4


def test_instruction_descriptor_f8f6f4(values):
    for M, N, v in values["idesc_e4m3_f32"]:
        check_idesc_common(v, M, N)
        assert field(v, 4, 2) == 1      # D: F32
        assert field(v, 16, 1) == 0     # B K-major
        assert field(v, 23, 1) == 0 and field(v, 29, 3) == 0 and field(v, 6, 1) == 0


def test_instruction_descriptor_b_major(values):
    rows = values["idesc_e4m3_f32_major"]
    assert len(rows) == 12
    for M, N, b, v in rows:
        check_idesc_common(v, M, N)
        assert field(v, 4, 2) == 1
        assert field(v, 16, 1) == b
        assert field(v, 23, 1) == 0 and field(v, 29, 3) == 0


def test_instruction_descriptor_block_scaled(values):
    rows = values["idesc_e4m3_bs"]
    assert len(rows) == 24
    for M, N, sf_id, v in rows:
        check_idesc_common(v, M, N)
        assert field(v, 4, 2) == sf_id  # B scale-factor id
        assert field(v, 16, 1) == 0
        assert field(v, 23, 1) == 1     # UE8M0 scale factors
        assert field(v, 29, 2) == sf_id  # A scale-factor id
        assert field(v, 31, 1) == 0 and field(v, 6, 1) == 0
