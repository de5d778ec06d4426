"""Pins of the oracle's KV-cache INT8 ("27届大模型面试准备（十九）…" sec. 6):
V per token (the page's quant_kv_per_token), K per channel over the tokens of a
head; hand-worked rows and columns, the independence each granularity implies,
the s/2 error bound, and the page's reason for per-channel K."""
import numpy as np

import oracle


def test_v_per_token_hand_rows():
    V = np.zeros((1, 3, 8), np.float32)
    V[0, 0] = [127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -127.0, 3.25]   # scale 1: half to even
    V[0, 1] = [254.0, 1.0, 3.0, 5.0, -2.0, 0.0, 0.0, 0.0]         # scale 2
    K = np.ones((1, 3, 8), np.float32)
    qk, sk, qv, sv, st = oracle.quant_kv(K, V)
    assert st == oracle.OK
    assert sv.tolist() == [[1.0, 2.0, np.float32(1e-8)]]          # an all-zero token clamps to 1e-8
    assert qv[0, 0].tolist() == [127, 0, 2, 2, 0, -2, -127, 3]
    assert qv[0, 1].tolist() == [127, 0, 2, 2, -1, 0, 0, 0]
    assert qv[0, 2].tolist() == [0] * 8


def test_k_per_channel_hand_columns():
    K = np.zeros((2, 4, 2), np.float32)
    K[0, :, 0] = [127.0, -63.5, 1.0, 0.5]      # channel 0 of head 0: scale 1
    K[0, :, 1] = [2.0, -4.0, 254.0, 3.0]       # channel 1 of head 0: scale 2
    K[1, :, 0] = [-12.7, 0.0, 6.35, 1.27]      # head 1 has its own scales
    K[1, :, 1] = 0.0
    qk, sk, qv, sv, st = oracle.quant_kv(K, np.zeros_like(K))
    assert st == oracle.OK
    assert sk[0].tolist() == [1.0, 2.0]
    assert qk[0, :, 0].tolist() == [127, -64, 1, 0]
    assert qk[0, :, 1].tolist() == [1, -2, 127, 2]
    assert sk[1, 0] == np.float32(np.float32(12.7) / np.float32(127.0))
    assert sk[1, 1] == np.float32(1e-8) and qk[1, :, 1].tolist() == [0, 0, 0, 0]


def _outlier_kv(seed):
    rng = np.random.default_rng(seed)
    Kc = rng.standard_normal((4, 256, 128)).astype(np.float32)
    Vc = rng.standard_normal((4, 256, 128)).astype(np.float32)
    Kc[:, :, [3, 40, 77, 101]] *= 50.0          # channel-wise outliers in K
    return Kc, Vc


def test_granularity_independence():
    """Scaling one channel of K moves only that channel's codes; scaling one
    token of V moves only that token's codes (a swapped axis fails both)."""
    Kc, Vc = _outlier_kv(1)
    qk0, _, qv0, _, _ = oracle.quant_kv(Kc, Vc)
    K2, V2 = Kc.copy(), Vc.copy()
    K2[:, :, 5] *= 100.0
    V2[:, 9, :] *= 100.0
    qk1, _, qv1, _, _ = oracle.quant_kv(K2, V2)
    ch = np.ones(128, bool)
    ch[5] = False
    tok = np.ones(256, bool)
    tok[9] = False
    assert np.array_equal(qk0[:, :, ch], qk1[:, :, ch])
    assert np.array_equal(qv0[:, tok, :], qv1[:, tok, :])


def test_error_within_half_a_step():
    Kc, Vc = _outlier_kv(2)
    qk, sk, qv, sv, st = oracle.quant_kv(Kc, Vc)
    assert st == oracle.OK
    assert np.all(np.abs(Kc - qk * sk[:, None, :]) <= sk[:, None, :] / 2 * (1 + 1e-6))
    assert np.all(np.abs(Vc - qv * sv[:, :, None]) <= sv[:, :, None] / 2 * (1 + 1e-6))


def test_per_channel_k_beats_per_token_on_outlier_channels():
    """Sec. 6's reason: with channel-wise outliers in K, one scale per channel
    keeps the ordinary channels precise; one scale per token does not."""
    Kc, _ = _outlier_kv(3)
    qk, sk, _, _, _ = oracle.quant_kv(Kc, Kc)
    e_ch = np.linalg.norm(Kc - qk * sk[:, None, :]) / np.linalg.norm(Kc)
    _, _, qt, st_, _ = oracle.quant_kv(Kc, Kc)   # V path = per token on the same tensor
    e_tok = np.linalg.norm(Kc - qt * st_[:, :, None]) / np.linalg.norm(Kc)
    normal = np.ones(128, bool)
    normal[[3, 40, 77, 101]] = False
    e_ch_n = np.linalg.norm((Kc - qk * sk[:, None, :])[:, :, normal])
    e_tok_n = np.linalg.norm((Kc - qt * st_[:, :, None])[:, :, normal])
    assert e_ch_n < 0.1 * e_tok_n, (e_ch_n, e_tok_n)
    assert e_ch <= e_tok
