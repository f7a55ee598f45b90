"""Host-side arithmetic of bench.py, checked on CPU: the algorithmic bytes and
FLOPs behind every roofline fraction against the figures derived for the
workloads from the layer's shapes (weights of every touched expert streamed
once, plus x, router tensors and out), the kernel count the JSON line
claims, and that a DRAM traffic figure is reported only from a profile
whose recorded source hash is the current kernel's."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_diffusion_moe_router_b200 import inputs  # noqa: E402

W = inputs.WORKLOADS


def test_bf16_canvas_bytes_and_flops():
    """One canvas layer with all 128 experts touched: 3 f d bf16 weights per
    expert (11,894,784 B), x in and out (1,441,792 B each), router weight,
    gamma (fp32); FLOPs 2 * 3 f d per token-expert pair plus the router's
    2 T E d."""
    w = W["canvas"]
    expert, step, flops, wbytes = bench.layer_costs(w, 128, w.T)
    assert wbytes == 3 * 704 * 2816 * 2 == 11_894_784
    assert expert == 128 * 11_894_784 == 1_522_532_352
    assert step == 1_522_532_352 + 2 * 256 * 2816 * 2 + 128 * 2816 * 4 + 2816 * 4
    assert step == 1_526_868_992
    assert flops == 256 * 8 * 2 * 3 * 704 * 2816 + 2 * 256 * 128 * 2816 == 24_545_067_008


def test_encode_and_int4_bytes():
    """T=2048 moves eight times the activations; the int4 layer streams half
    a byte per weight plus fp16 group scales (22 groups along d, 6 along f)."""
    w = W["encode"]
    _, step, flops, _ = bench.layer_costs(w, 128, w.T)
    assert step == 1_522_532_352 + 2 * 2048 * 2816 * 2 + 128 * 2816 * 4 + 2816 * 4
    assert step == 1_547_054_080
    assert flops == 2048 * 8 * 2 * 3 * 704 * 2816 + 2 * 2048 * 128 * 2816
    w4 = W["canvas4"]
    assert (w4.n_groups_d, w4.n_groups_f) == (22, 6)
    _, step4, _, wb4 = bench.layer_costs(w4, 128, w4.T)
    assert wb4 == 3 * 704 * 2816 // 2 + 2 * (2 * 704 * 22 + 2816 * 6)
    assert step4 == 397_224_960


def test_fp8_and_fp4_bytes():
    """fp8: one byte per weight and one fp32 scale per weight row; fp4: half
    a byte per weight, one E4M3 scale per 16 weights and one fp32 scale per
    row."""
    _, _, _, wb8 = bench.layer_costs(W["canvas8"], 128, 256)
    assert wb8 == 3 * 704 * 2816 + 4 * (2 * 704 + 2816) == 5_964_288
    _, _, _, wb4f = bench.layer_costs(W["canvas4f"], 128, 256)
    assert wb4f == 3 * 704 * 2816 // 2 + 2 * 704 * (4 + 2816 // 16) + 2816 * (4 + 704 // 16)
    assert wb4f == 3_362_304


def test_stack_layer_bytes_count_the_residual_and_bias():
    """A stack layer also reads the residual and the router bias."""
    w = W["stack30"]
    _, step, _, _ = bench.layer_costs(w, 77, w.T)
    assert step == 77 * 11_894_784 + 3 * 256 * 2816 * 2 + 128 * 2816 * 4 + 2816 * 4 + 128 * 4


@pytest.mark.parametrize("name,T,n", [("canvas", 256, 4), ("stack30", 256, 4),
                                      ("canvas8", 256, 4), ("encode", 2048, 5)])
def test_launches_per_layer(name, T, n):
    """Router, plan + gather (one launch for one canvas, two above), expert
    kernel, combine."""
    assert bench.launches_per_layer(W[name], T, "auto") == n


def test_traffic_only_from_a_profile_of_the_current_kernel():
    """Every committed expert-kernel profile records the hash of the sources
    it was taken from; each matches the current sources, so the bench's
    traffic figure is the profiled kernel's."""
    for name, (fname, _) in bench.PROFILES.items():
        text = open(os.path.join(ROOT, "profiles", fname)).read()
        recorded = [ln.split(":", 1)[1].strip() for ln in text.splitlines()
                    if ln.startswith("source_sha256_16:")]
        assert recorded == [bench.source_hash(name)], name
        assert bench.recorded_traffic(name) > 0, name
