"""Host-side arithmetic of the bench line, on CPU: the algorithmic work the
roofline divides by, the roofline itself, and the staleness rule that drops a
DRAM-traffic figure once the kernel's sources change."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_bench_workload_is_the_res_block():
    assert (bench.H, bench.W, bench.C, bench.BLOCK) == (256, 256, 128, 8)


def test_conv_work_per_tile():
    # one 8x8 tile of the 3x3, 128 -> 128 conv: 64 px x 128 x 128 x 9 MACs;
    # a 10x10x128 bf16 halo in, an 8x8x128 bf16 tile out (and as much residual)
    flops1, bytes1 = bench.conv_work(1, residual=False)
    flops2, bytes2 = bench.conv_work(2, residual=False)
    assert flops2 - flops1 == 2 * 64 * 128 * 128 * 9 == 18_874_368
    assert bytes2 - bytes1 == 10 * 10 * 128 * 2 + 8 * 8 * 128 * 2 == 25_600 + 16_384
    weights = 128 * 9 * 128 * 2 + 128 * 4      # bf16 KRSC + float bias
    assert bytes1 - (bytes2 - bytes1) == weights
    _, bres2 = bench.conv_work(2, residual=True)
    _, bres1 = bench.conv_work(1, residual=True)
    assert bres2 - bres1 == 25_600 + 2 * 16_384
    # the bench's 51 tiles
    f, b = bench.conv_work(51, residual=False)
    assert f == 51 * 18_874_368 and b == 51 * 41_984 + weights


def test_resblock_work_per_tile():
    # both convs' MACs on an 8x8 tile (the recomputed ring of y1 is not
    # counted); the 12x12x128 bf16 halo of x read once (it holds the residual);
    # y1 and out written at the tile
    f1, b1 = bench.resblock_work(1)
    f2, b2 = bench.resblock_work(2)
    assert f2 - f1 == 2 * 18_874_368
    assert b2 - b1 == 12 * 12 * 128 * 2 + 2 * 8 * 8 * 128 * 2 == 36_864 + 32_768
    fixed = 2 * (128 * 9 * 128 * 2) + 6 * 128 * 4       # two weight tensors, biases and GroupNorm affines
    assert b1 - (b2 - b1) == fixed
    assert f1 - (f2 - f1) == 0


def test_step_work():
    # the one-launch step: both inputs once, y1 and out at the tiles, both
    # weight tensors, and the list; the MACs of both convs on the tiles
    f, b = bench.step_work(51)
    assert f == 51 * 2 * 18_874_368
    fixed = 2 * (128 * 9 * 128 * 2) + 6 * 128 * 4
    assert b == 33_554_436 + 51 * 8 + 51 * 2 * 16_384 + fixed


def test_mask_work():
    # both 256x256x128 bf16 activations read once, the list written
    assert bench.mask_work(0) == 2 * 256 * 256 * 128 * 2 + 4 == 33_554_436
    assert bench.mask_work(51) - bench.mask_work(0) == 51 * 8


def test_layer_roofline():
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    # compute-bound bf16 layer: 1e9 MACs -> 2 GFLOP / 1 PFLOP/s = 2 us
    r = bench.layer_roofline(1e9, 1e3, 16, peaks, 4.0)
    assert r["bound"] == "tensor" and r["roof_us"] == pytest.approx(2.0) and r["frac"] == pytest.approx(0.5)
    # byte-bound: 5e6 bytes / 5 TB/s = 1 us
    r = bench.layer_roofline(1e3, 5e6, 16, peaks, 10.0)
    assert r["bound"] == "hbm" and r["roof_us"] == pytest.approx(1.0) and r["frac"] == pytest.approx(0.1)
    # float32 layers go against the FP32 FMA peak: 148 SMs x 128 lanes x 2 x 1.965 GHz
    assert bench.FP32_ALU_TFLOPS == pytest.approx(74.45, rel=1e-3)
    r = bench.layer_roofline(74.45e6 / 2, 1.0, 32, peaks, 2.0)
    assert r["bound"] == "alu" and r["roof_us"] == pytest.approx(1.0, rel=1e-3)


def test_traffic_dropped_when_code_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("// first version\nint f() { return 1; }\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"sources": ["k.cu"], "code_sha": bench.code_sha(["k.cu"]), "bytes_per_launch": 1234}
    (prof / "ncu_traffic.json").write_text(json.dumps({"k_test": entry}))
    assert bench.ncu_traffic("k_test") == 1234.0
    assert bench.ncu_traffic("k_other") is None
    # comments and blank lines do not change the kernel
    src.write_text("/* reworded */\n\nint f() { return 1; }  // same code\n")
    assert bench.ncu_traffic("k_test") == 1234.0
    # code does
    src.write_text("int f() { return 2; }\n")
    assert bench.ncu_traffic("k_test") is None
    os.remove(src)
    assert bench.ncu_traffic("k_test") is None


def test_strip_c_comments():
    t = ('int a = 1; // one\n/* two\n lines */ int b = 2; char c = \'/\';\n'
         'const char *s = "// kept /* kept */";\n\n  x = a/*in*/+b;\n')
    assert bench.strip_c_comments(t) == ('int a = 1;\n  int b = 2; char c = \'/\';\n'
                                         'const char *s = "// kept /* kept */";\n  x = a +b;')


def test_bench_workload_tiles_from_the_oracle(orc):
    # the bench's edit (seed 0, 1.2% of the pixels) activates 51 of the 1024
    # 8x8 tiles after one-tile dilation, as its JSON line reports
    from spatially_sparse_incremental_b200 import inputs
    blk = inputs.make_cfg3(0, H=bench.H, W=bench.W, C=bench.C, area=0.012, block=bench.BLOCK)
    tiles = orc.reduce_mask(blk.x_orig, blk.x_edit, bench.THRESH, [(bench.H, bench.W, bench.BLOCK)], 1)[0]
    assert len(tiles) == 51
    edited = orc.pixel_mask(blk.x_orig, blk.x_edit, bench.THRESH).mean()
    assert abs(edited - 0.012) < 0.002
