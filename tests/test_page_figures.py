"""Host-side pins against figures the pages print (CPU only)."""
import json
import math
from pathlib import Path

import pytest
import torch

from selective_state_space_55_b200 import inputs as I
from selective_state_space_55_b200 import roofline as R

FIG = json.loads((Path(__file__).parent / "golden" / "page_figures.json").read_text())


def test_state_numbers_match_page():
    f = FIG["mamba_2p8b_state_numbers"]
    n = R.state_numbers(f["layers"], f["channels"], f["dstate"], f["conv_taps"])
    assert n == f["value"]
    assert round(n * 2 / 1e6, 1) == FIG["mamba_2p8b_state_mb_16bit"]["value"]


def test_kv_cache_bytes_match_page():
    f = FIG["pythia_2p8b_kv_bytes_per_token"]
    per_tok = R.kv_cache_bytes_per_token(f["layers"], f["width"], f["bytes_per_number"])
    assert per_tok == f["value"]
    tokens = FIG["pythia_2p8b_kv_mb_2048_tokens"]["tokens"]
    assert round(per_tok * tokens / 1e6) == FIG["pythia_2p8b_kv_mb_2048_tokens"]["value"]
    state_bytes = 2 * R.state_numbers(64, 5120, 16, 4)
    first = math.ceil(state_bytes / per_tok)
    assert first == FIG["kv_exceeds_state_at_token"]["value"]
    assert int(per_tok * tokens / state_bytes) == FIG["kv_over_state_at_2048"]["value"]


def test_update_bytes_decode_shape():
    # 128 x 4096 chains x 16 fp32 state entries, read and written.
    b = R.update_bytes(128, 4096, 16)
    assert b - 2 * 128 * 4096 * 16 * 4 == 128 * 4096 * 2 * 4 + 2 * 128 * 16 * 2 + 4096 * 16 * 4 + 2 * 4096 * 4


def test_scan_mufu_model():
    assert R.scan_mufu_per_element(16) == 20
    assert R.scan_mufu_per_element(16, has_z=False, softplus=False) == 16
    assert R.scan_mufu_per_element(16, io_bytes=2) == 19          # bf16: lg2 softplus, tanh gate
    assert R.scan_mufu_per_element(16, io_bytes=2, zoh=True) == 20  # + 1/Delta
    peak = R.mufu_peak_elements_per_s(148, 1965.0, 20)
    assert abs(peak / 1e9 - 232.7) < 0.1


def test_a_init_is_s4d_real():
    lo, hi = FIG["a_init_range"]["value"]
    A = I.s4d_real_A(3, 16)
    assert A[0, 0].item() == lo and A[0, -1].item() == hi
    assert torch.equal(A[1], A[0])


def test_layer_bias_recipe_lands_in_range():
    # the layer-shape recipe draws softplus(bias) uniformly from [1e-3, 0.1]
    lo, hi = 1e-3, 0.1
    g = torch.Generator().manual_seed(0)
    bias = I.layer_delta_bias(4096, g, "cpu").double()
    sp = torch.nn.functional.softplus(bias)
    assert sp.min().item() >= lo * (1 - 1e-6) and sp.max().item() <= hi * (1 + 1e-6)


def test_dna_inputs_take_four_symbols():
    cfg = I.SCAN_CONFIGS["long_dna_1m"].resized(dim=64, seqlen=512)
    x = I.make_scan_inputs(cfg, "cpu", seed=0)
    cols = {tuple(x["u"][0, :, t].tolist()) for t in range(512)}
    assert len(cols) == 4


@pytest.mark.parametrize("name", sorted(I.SCAN_CONFIGS))
def test_configs_shapes(name):
    c = I.SCAN_CONFIGS[name]
    small = c.resized(batch=min(c.batch, 2), dim=min(c.dim, 64), seqlen=min(c.seqlen, 64))
    x = I.make_scan_inputs(small, "cpu", seed=0)
    assert x["u"].shape == (small.batch, small.dim, small.seqlen)
    assert x["B"].shape == (small.batch, small.dstate, small.seqlen)
    assert x["u"].dtype == c.io_dtype and x["B"].dtype == c.bc_dtype
    assert x["A"].dtype == torch.float32 and x["A"].shape == (small.dim, small.dstate)


def test_mamba2_layer_byte_and_flop_counts():
    """The Mamba-2 layer's algorithmic bytes and issued tensor FLOPs on the 2.7B
    layer shape, counted by hand: per (token, head) x, z, out (64 bf16 each) and
    dt (one bf16); per token B and C (128 bf16 each, one group); the final fp32
    state of every head; per 128-token chunk and head four dense products, three
    of them issued twice (hi and lo halves of a computed operand)."""
    from selective_state_space_55_b200 import roofline as R
    batch, L, H, P, N, Q = 16, 2048, 80, 64, 128, 128
    tokens = batch * L
    by_hand = tokens * H * (3 * P * 2 + 2) + tokens * 2 * N * 2 + batch * H * P * N * 4
    assert by_hand == 1_070_596_096
    assert R.ssd_bytes(batch, L, H, P, 1, N) == by_hand
    chunks = L // Q
    products = Q * Q * N + Q * Q * P + N * Q * P + Q * N * P   # C B^T, Gm x, B^T Xw, C H^T
    assert R.ssd_chunk_flops(batch, L, H, P, N, Q) == 2 * products * batch * H * chunks
    assert R.ssd_chunk_flops(batch, L, H, P, N, Q) / (tokens * H * P) == 1280
    # issued: the products of Gm x, B^T Xw and C H^T twice (hi and lo operands)
    issued = Q * Q * N + 2 * (Q * Q * P + N * Q * P + Q * N * P)
    assert R.ssd_issued_flops(batch, L, H, P, N, Q) == 2 * issued * batch * H * chunks
    assert R.ssd_issued_flops(batch, L, H, P, N, Q) / (tokens * H * P) == 2048
