"""The codec quality / bit-rate report (decode_attention_rand_b200.quality).

Bit accounting (CPU): the abstract of "TurboAngle: Near-Lossless KV Cache
Compression via Uniform Angle Quantization" gives 3.28-3.67 angle bits per
element for its early-boost schedules and 6.56 total bits per element on
Mistral-7B; the accounting here (log2 L per pair of elements, 8-bit K and
4-bit V norms per pair, fp16 per-vector parameters) must land the
Mistral-shaped schedule inside that angle range and near that total, and the
stored rows must take exactly the nominal bits when every L is a power of 2.

Errors (GPU): the tool's dequantization error equals the oracle's on the
same data, and every error falls as the codebook grows.
"""
import math

import numpy as np
import pytest

from decode_attention_rand_b200 import kvq, quality, synth


def test_bits_per_element_llama_layer():
    b = quality.bits_per_element(128, 128, 64)
    assert b["angle"] == pytest.approx(3.25)
    assert b["norms"] == pytest.approx(3.0)
    assert b["params"] == pytest.approx(48 / 256)
    assert b["total"] == pytest.approx(3.25 + 3.0 + 0.1875)
    # 122 + 84 stored bytes per token and KV head, 2 x 128 elements
    assert b["stored"] == pytest.approx(206 * 8 / 256)
    assert b["stored"] == pytest.approx(b["total"])


def test_stored_bits_round_angle_words_up():
    # L = 200 needs 8 bits per code but log2(200) = 7.64 nominal bits
    b = quality.bits_per_element(128, 200, 200)
    assert b["angle"] == pytest.approx(math.log2(200) / 2)
    assert b["stored"] > b["total"]
    assert b["stored"] == pytest.approx((8 / 2 + 3.0 + 0.1875))


def test_mistral_schedule_inside_the_abstract_range():
    w = synth.WORKLOADS["mistral7b_32layers_b8_hq32_hkv8_d128_ctx32768"]
    s = quality.schedule_bits(w)
    assert s["angle"] == pytest.approx((4 * 4.0 + 28 * 3.25) / 32)
    assert 3.28 <= s["angle"] <= 3.67
    assert s["total"] == pytest.approx(s["angle"] + 3.0 + 0.1875)
    assert abs(s["total"] - 6.56) < 0.05


def test_tinyllama_schedule():
    w = synth.WORKLOADS["tinyllama_22layers_b4_hq32_hkv4_d64_ctx65536"]
    s = quality.schedule_bits(w)
    assert s["angle"] == pytest.approx((2 * 4.0 + 20 * (7 + 5) / 4) / 22)
    assert s["params"] == pytest.approx(48 / 128)


@pytest.mark.gpu
def test_codec_error_matches_oracle_and_falls_with_L():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import oracle as O
    from decode_attention_rand_b200 import build as kbuild
    kbuild.build()
    w = synth.WORKLOADS["tiny_b1_hq4_hkv2_d128_ctx256"]
    rows = [quality.codec_error(w, 0, L, L) for L in (32, 64, 256)]
    for a, b in zip(rows, rows[1:]):
        assert b["k_rel_l2_mean"] < a["k_rel_l2_mean"]
        assert b["attn_rel_l2_mean"] < a["attn_rel_l2_mean"]
    # the same numbers from the oracle's codec on the same input
    sk, sv = synth.layer_signs(w, 0)
    # the tool draws its inputs on the GPU; the same draw, moved to the host
    k = synth.kv(w, 0, synth.KIND_K, device="cuda").cpu().numpy()
    v = synth.kv(w, 0, synth.KIND_V, device="cuda").cpu().numpy()
    for r in rows:
        for x, s, mode, key in ((k, sk, O.MODE_LIN8, "k_rel_l2_mean"),
                                (v, sv, O.MODE_LOG4, "v_rel_l2_mean")):
            xh = O.dequant(O.encode(x, s, r["L_K"], mode), s).reshape(x.shape)
            xd = x.astype(np.float64).reshape(-1, x.shape[-1])
            e = np.linalg.norm(xh.reshape(-1, x.shape[-1]) - xd, axis=1) / np.linalg.norm(xd, axis=1)
            # the GPU rounds its dequantized vectors to fp16
            assert r[key] == pytest.approx(e.mean(), rel=2e-3, abs=2e-4), (key, r["L_K"])


def test_bits_per_element_other_norm_modes():
    """4-bit log K norms (and 8-bit linear V norms) count 4 (8) bits per pair
    and carry their own fp16 parameters: LOG4 two per vector, LIN8 one."""
    lin, log = kvq.KVQ_NORM_LIN8, kvq.KVQ_NORM_LOG4
    b = quality.bits_per_element(128, 128, 64, log, log)
    assert b["norms"] == pytest.approx((4 + 4) / 4)
    assert b["params"] == pytest.approx((32 + 32) / 256)
    assert b["stored"] == pytest.approx(b["total"])
    b = quality.bits_per_element(64, 128, 64, log, lin)
    assert b["norms"] == pytest.approx((4 + 8) / 4)
    assert b["params"] == pytest.approx((32 + 16) / 128)
    assert b["stored"] == pytest.approx(b["total"])


@pytest.mark.gpu
@pytest.mark.parametrize("mk,mv", [(kvq.KVQ_NORM_LOG4, kvq.KVQ_NORM_LOG4),
                                   (kvq.KVQ_NORM_LOG4, kvq.KVQ_NORM_LIN8)])
def test_norm_mode_sweep_matches_oracle(mk, mv):
    """The other norm pairings, at a codebook past 256: the tool's
    dequantization errors equal the oracle's, and the attention error (the
    decode kernels now take every codec) is reported."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import oracle as O
    from decode_attention_rand_b200 import build as kbuild
    kbuild.build()
    w = synth.WORKLOADS["tiny_b1_hq4_hkv2_d128_ctx256"]
    r = quality.codec_error(w, 0, 1024, 1024, mode_k=mk, mode_v=mv)
    assert r["attn_rel_l2_mean"] is not None and r["attn_rel_l2_mean"] < 0.5
    sk, sv = synth.layer_signs(w, 0)
    k = synth.kv(w, 0, synth.KIND_K, device="cuda").cpu().numpy()
    v = synth.kv(w, 0, synth.KIND_V, device="cuda").cpu().numpy()
    for x, s, mode, key in ((k, sk, mk, "k_rel_l2_mean"), (v, sv, mv, "v_rel_l2_mean")):
        xh = O.dequant(O.encode(x, s, 1024, mode), s).reshape(x.shape)
        xd = x.astype(np.float64).reshape(-1, x.shape[-1])
        e = np.linalg.norm(xh.reshape(-1, x.shape[-1]) - xd, axis=1) / np.linalg.norm(xd, axis=1)
        assert r[key] == pytest.approx(e.mean(), rel=2e-3, abs=2e-4), key
