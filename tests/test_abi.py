"""CPU checks of the C ABI: the library loads, exports every symbol the header
declares, validates its arguments on the host and sizes the state as the page's
memory formula says ("MicroAdam (Sparse-Gradient Adaptive Optimization with
Quantized Error Feedback)", paragraph 2). No compute call is made here."""
import ctypes
import json
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mua.h")


@pytest.fixture(scope="module")
def mua():
    from compressed_state_optimizer_b200 import build
    build.build()
    from compressed_state_optimizer_b200 import binding
    return binding


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mua_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported(mua):
    names = declared_symbols()
    assert len(names) >= 13
    lib = mua.library()
    for n in names:
        assert hasattr(lib, n), n
        assert n in mua.SIGNATURES, n
    out = subprocess.run(["nm", "-D", "--defined-only", mua.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mua_[a-z0-9_]+)\b", out))
    assert set(names) <= exported
    assert all(n in names for n in mua.SIGNATURES)


def test_built_for_sm100a(mua):
    out = subprocess.run(["cuobjdump", "--list-elf", mua.library_path()],
                         capture_output=True, text=True)
    if out.returncode == 0:
        assert "sm_100a" in out.stdout


def _create(mua, *args):
    h = ctypes.c_void_p()
    rc = mua.library().mua_create(*args, ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("args,code", [
    ((0, 16384, 164, 10, 4), -1),          # d < 1
    ((100, 32767, 164, 10, 4), -1),        # B_d >= 2^15 - 1
    ((100, 16383, 164, 10, 4), -1),        # odd B_d
    ((100, 16384, 0, 10, 4), -1),          # k_b < 1
    ((100, 16384, 16385, 10, 4), -1),      # k_b > B_d
    ((100, 16384, 164, 0, 4), -1),         # m < 1
    ((100, 16384, 164, 65, 4), -1),        # m > 64
    ((100, 16384, 164, 10, 8), -2),        # b != 4
    ((100, 16384, 16384, 10, 4), -2),      # window of a block too large for the chip
    ((100, 16384, 1537, 10, 4), -2),       # m * kp = 15400 > 15360
])
def test_create_rejects(mua, args, code):
    rc, h = _create(mua, *args)
    assert rc == code and not h.value
    assert mua.strerror(rc)


def test_create_accepts_limits(mua):
    for args in [(1, 2, 1, 1, 4), (32766 * 3 + 5, 32766, 328, 10, 4), (10**12, 16384, 164, 64, 4),
                 (100, 32766, 1536, 10, 4)]:
        rc, h = _create(mua, *args)
        assert rc == 0 and h.value
        mua.library().mua_destroy(h)


def test_state_bytes_and_layout(mua):
    m = mua.MicroAdam(1000, block_size=256, k_per_block=3, window=5)
    nb = 4
    assert m.layout.blocks == nb and m.layout.row_stride == 4
    assert m.layout.codes == 256 and m.layout.window == 256 + 512
    assert m.state_bytes == 256 + 512 + 4 * nb * 5 * 4 == m.layout.bytes
    assert m.d == 1000 and m.offset == 0


def test_state_memory_matches_page(mua):
    """The state of the LLaMA-2-7B-shaped vector at m = 10, k = 1 %: 0.5 d + 4 m k
    bytes, the page's 5.65 GB (GiB) against 12.55 for 8-bit and 50.21 for fp32
    AdamW; and the break-even window m_max = 37.5."""
    gold = json.load(open(os.path.join(ROOT, "tests", "golden", "microadam_memory.json")))
    d = gold["llama2_7b_param_count_from_shapes"]
    from compressed_state_optimizer_b200 import workloads
    assert workloads.numel(workloads.llama2_7b_shapes()) == d
    m = mua.MicroAdam(d, block_size=16384, k_per_block=164, window=10)
    printed = gold["printed"]
    gib = 2.0 ** 30
    assert round(m.state_bytes / gib, 2) == printed["microadam_state_at_m10"]["value"]
    assert round(0.9 * d / gib, 2) == printed["microadam_state_at_m10"]["value"]
    assert round(2 * d / gib, 2) == printed["adamw_8bit_state"]["value"]
    assert round(8 * d / gib, 2) == printed["adamw_fp32_state"]["value"]
    nb = -(-d // 16384)
    assert m.state_bytes == 256 + -(-((d + 1) // 2) // 256) * 256 + 4 * nb * 10 * 164
    # k_b = ceil(16384/100) = 164 keeps 0.098 % more entries than k = d/100.
    paper = 0.5 * d + 4 * 10 * d / 100
    assert 0 < (m.state_bytes - paper) / d < 4 * 10 * (164 / 16384 - 0.01) + 1e-6
    # 0.5 d + 4 m d/100 < 2 d  <=>  m < 37.5
    assert all((0.5 + 0.04 * mm < 2.0) == (mm < printed["m_max"]) for mm in range(1, 80))


# The calls below pass fake device addresses and rely on the host-side checks
# returning first. They run in a child process that sees no GPU
# (CUDA_VISIBLE_DEVICES=""), so a regression in those checks makes a CUDA call
# fail there instead of launching a kernel on a wild address.
_HIDDEN_PRELUDE = """
import ctypes, sys
sys.path.insert(0, {root!r})
from compressed_state_optimizer_b200 import binding as mua
lib = mua.library()
m = mua.MicroAdam(64, block_size=32, k_per_block=2, window=2)
ok, bad = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1008)
"""


def _run_without_gpu(body: str):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    code = _HIDDEN_PRELUDE.format(root=ROOT) + body
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr


@pytest.mark.parametrize("t,lr,b1,b2,eps,code", [
    (0, 1e-3, 0.9, 0.999, 1e-8, -1),
    (1, float("nan"), 0.9, 0.999, 1e-8, -1),
    (1, 1e-3, 1.0, 0.999, 1e-8, -1),
    (1, 1e-3, 0.9, -0.1, 1e-8, -1),
    (1, 1e-3, 0.9, 0.999, -1.0, -1),
    (1, 1e-3, 0.9, 0.999, 0.0, -1),    # eps = 0 would divide 0 by 0 on all-zero windows
])
def test_step_validates_before_any_cuda_call(mua, t, lr, b1, b2, eps, code):
    _run_without_gpu(f"""
rc = lib.mua_step(m._h, ok, ok, ok, {lr!r}, {b1!r}, {b2!r}, {eps!r}, 0.0, {t}, 1, None)
assert rc == {code}, rc
""".replace("nan", "float('nan')"))


def test_step_rejects_null_and_misaligned(mua):
    _run_without_gpu("""
assert lib.mua_step(m._h, None, ok, ok, 1e-3, .9, .999, 1e-8, 0., 1, 1, None) == -1
assert lib.mua_step(m._h, bad, ok, ok, 1e-3, .9, .999, 1e-8, 0., 1, 1, None) == -3
assert lib.mua_select(m._h, ok, ok, bad, 1e-3, .9, .999, 1e-8, 0., 1, 1, None, None,
                      None) == -3
assert lib.mua_apply(m._h, ok, ok, ok, 1e-3, .9, .999, 1e-8, 0., 0, 1, None, None,
                     None) == -1
assert lib.mua_step(None, ok, ok, ok, 1e-3, .9, .999, 1e-8, 0., 1, 1, None) == -1
out = ctypes.c_int32()
assert lib.mua_get_status(m._h, None, None, ctypes.byref(out)) == -1
assert lib.mua_get_status(m._h, ok, None, None) == -1
assert lib.mua_get_status(None, ok, None, ctypes.byref(out)) == -1
""")


def test_minmax_offset(mua):
    m = mua.MicroAdam(64, block_size=32, k_per_block=2, window=2)
    lib = mua.library()
    assert lib.mua_minmax_offset(m._h, 0) == -1
    assert lib.mua_minmax_offset(m._h, 1) in (0, 8)
    assert lib.mua_minmax_offset(m._h, 1) != lib.mua_minmax_offset(m._h, 2)
    assert lib.mua_minmax_offset(None, 1) == -1


def test_shard_geometry(mua):
    d, Bd = 10 * 64 + 17, 64
    whole = mua.MicroAdam(d, block_size=Bd, k_per_block=2, window=3)
    a = mua.MicroAdam(d, block_size=Bd, k_per_block=2, window=3, shard=(0, 6))
    b = mua.MicroAdam(d, block_size=Bd, k_per_block=2, window=3, shard=(6, 5))
    assert a.d + b.d == d and b.offset == 6 * Bd
    assert a.layout.blocks + b.layout.blocks == whole.layout.blocks
    with pytest.raises(mua.MuaError):
        mua.MicroAdam(d, block_size=Bd, k_per_block=2, window=3, shard=(6, 6))


def _create_seg(mua, segs, Bd=256, kb=3, m=5, bits=4):
    import ctypes
    lib = mua.library()
    h = ctypes.c_void_p()
    arr = (ctypes.c_int64 * max(1, len(segs)))(*segs)
    rc = lib.mua_create_segmented(arr, len(segs), Bd, kb, m, bits, ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("segs,code", [
    ([], -1),                       # no tensor
    ([100, 0, 40], -1),             # empty tensor
    ([100, 37, 40], -2),            # odd length: a block would start inside a code byte
    ([2] * 513, -2),                # more than MUA_MAX_SEGMENTS
])
def test_create_segmented_rejects(mua, segs, code):
    rc, h = _create_seg(mua, segs)
    assert rc == code and not h.value


def test_segmented_layout(mua):
    """Blocks are counted tensor by tensor; the state is the flat layout of d with
    that block count."""
    segs = [1000, 256, 10, 512 + 2]
    m = mua.MicroAdam(sum(segs), block_size=256, k_per_block=3, window=5, segments=segs)
    nb = 4 + 1 + 1 + 3
    d = sum(segs)
    assert m.layout.blocks == nb == m.blocks and m.d == d
    codes_bytes = -(-((d + 1) // 2) // 256) * 256
    assert m.layout.window == 256 + codes_bytes
    assert m.state_bytes == 256 + codes_bytes + 4 * nb * 5 * 4 == m.layout.bytes
    with pytest.raises(ValueError):
        mua.MicroAdam(d + 2, block_size=256, k_per_block=3, window=5, segments=segs)
