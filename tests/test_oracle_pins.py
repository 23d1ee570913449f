"""Pins of the CPU oracle against what the model pages and mathematics fix.

Each test checks the oracle against something other than itself: figures the
pages print (tests/golden/page_facts.json), closed forms, brute force on tiny
inputs, invariants, and PyTorch's own float64 layers where a step reduces to a
library routine (Conv1d, LayerNorm, GELU, scaled-dot-product attention,
TransformerEncoderLayer with norm_first).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S

torch.set_default_dtype(torch.float64)
RNG = np.random.default_rng(1234)


class Geo:
    """Minimal geometry object accepted by oracle.encode_clip."""

    def __init__(self, n_layers, n_heads, pool_step=1, proj_hidden=0, proj_out=0, ln_eps=1e-5, head_dim=64,
                 attn_chunk=0):
        self.n_layers, self.n_heads, self.pool_step = n_layers, n_heads, pool_step
        self.proj_hidden, self.proj_out, self.ln_eps, self.head_dim = proj_hidden, proj_out, ln_eps, head_dim
        self.attn_chunk = attn_chunk


# ------------------------------------------------------------------ counts
def test_page_counts(page_facts):
    pre = page_facts["whisper_preprocessor"]
    assert pre["chunk_length_s"] * pre["sampling_rate"] == pre["n_samples"]
    assert O.frames_for_seconds(pre["chunk_length_s"], pre["sampling_rate"], pre["hop_length"]) == pre["nb_max_frames"]
    assert O.encoder_positions(pre["nb_max_frames"]) == page_facts["audio_tokens_per_30s"]["positions"]
    assert O.encoder_positions(pre["nb_max_frames"]) == page_facts["whisper_large"]["max_source_positions"]
    mc = page_facts["minicpm_o_audio"]
    assert O.pooled_positions(1500, mc["audio_pool_step"]) == mc["approx_tokens_per_30s"]
    # the tiny 2 s case: 200 frames -> 100 positions
    assert O.frames_for_seconds(2.0) == 200 and O.encoder_positions(200) == 100


def test_head_geometry(page_facts):
    v = page_facts["voxtral_encoder"]
    assert v["heads"] * v["head_dim"] == v["hidden_size"] and v["kv_heads"] == v["heads"]
    mc = page_facts["minicpm_o_audio"]
    assert mc["encoder_attention_heads"] * 64 == mc["d_model"]
    for name in ("medium_pool", "large_b16"):
        cfg = S.CONFIGS[name]
        assert cfg.n_heads * cfg.head_dim == cfg.d_model


def test_weight_shapes_match_pages(page_facts):
    wl = page_facts["whisper_large"]
    cfg = S.CONFIGS["large_b16"]
    shapes = dict(S.weight_shapes(cfg))
    assert list(shapes["layers.0.q_w"]) == wl["q_proj_shape_layers_0_and_31"]
    assert list(shapes["layers.31.q_w"]) == wl["q_proj_shape_layers_0_and_31"]
    assert "layers.32.q_w" not in shapes
    assert shapes["conv1_w"] == (wl["d_model"], wl["num_mel_bins"], 3)
    assert shapes["layers.0.fc1_w"] == (wl["encoder_ffn_dim"], wl["d_model"])
    assert "layers.0.k_b" not in shapes           # k projection has no bias
    # Whisper-large encoder parameter count (position table excluded):
    # stem 5,409,280 + 32 x 19,676,160 + final LN 2,560
    assert sum(int(np.prod(s)) for _, s in S.weight_shapes(cfg)) == 635_048_960
    med = S.CONFIGS["medium_pool"]
    assert sum(int(np.prod(s)) for _, s in S.weight_shapes(med)) == 305_680_384
    pj = S.CONFIGS["large_proj_b32"]
    sh = dict(S.weight_shapes(pj))
    assert sh["proj1_w"] == (3072, 1280) and sh["proj2_w"] == (3072, 3072)


def test_positions_bruteforce():
    """conv2 (k3, s2, p1) positions = number of windows inside the padded clip."""
    for t in range(1, 3001):
        brute = sum(1 for j in range(t + 2) if 2 * j + 2 <= t + 1)   # window [2j, 2j+2] in padded [0, t+1]
        assert O.encoder_positions(t) == brute == -(-t // 2)
    for t in range(1, 41):
        x = RNG.standard_normal((2, t))
        assert O.conv1d(x, RNG.standard_normal((3, 2, 3)), None, 1).shape == (3, t)
        assert O.conv1d(x, RNG.standard_normal((3, 2, 3)), None, 2).shape == (3, O.encoder_positions(t))


# -------------------------------------------------------------------- conv
def _conv_brute(x, w, b, stride):
    c_in, t = x.shape
    t_out = (t + 2 - 3) // stride + 1
    y = [[0.0] * t_out for _ in range(w.shape[0])]
    for o, j in itertools.product(range(w.shape[0]), range(t_out)):
        acc = 0.0 if b is None else float(b[o])
        for c in range(c_in):
            for k in range(3):
                tt = stride * j + k - 1
                if 0 <= tt < t:
                    acc += float(w[o, c, k]) * float(x[c, tt])
        y[o][j] = acc
    return np.array(y)


@pytest.mark.parametrize("t", [1, 2, 5, 6])
@pytest.mark.parametrize("stride", [1, 2])
def test_conv1d_bruteforce(t, stride):
    x = RNG.standard_normal((2, t))
    w = RNG.standard_normal((3, 2, 3))
    b = RNG.standard_normal(3)
    np.testing.assert_allclose(O.conv1d(x, w, b, stride), _conv_brute(x, w, b, stride), rtol=0, atol=1e-13)


def test_conv1d_special_kernels():
    x = RNG.standard_normal((4, 9))
    centre = np.zeros((4, 4, 3)); centre[np.arange(4), np.arange(4), 1] = 1.0
    np.testing.assert_array_equal(O.conv1d(x, centre, None, 1), x)
    np.testing.assert_array_equal(O.conv1d(x, centre, None, 2), x[:, ::2])
    first = np.zeros((4, 4, 3)); first[np.arange(4), np.arange(4), 0] = 1.0   # y[j] = x[j-1]
    y = O.conv1d(x, first, None, 1)
    np.testing.assert_array_equal(y[:, 1:], x[:, :-1])
    np.testing.assert_array_equal(y[:, 0], 0.0)
    # single channel: numpy.correlate over the zero-padded signal
    x1 = RNG.standard_normal((1, 11)); w1 = RNG.standard_normal((1, 1, 3))
    ref = np.correlate(np.pad(x1[0], 1), w1[0, 0], mode="valid")
    np.testing.assert_allclose(O.conv1d(x1, w1, None, 1)[0], ref, atol=1e-14)


def test_conv1d_matches_torch():
    x = RNG.standard_normal((5, 17))
    for stride in (1, 2):
        w = RNG.standard_normal((6, 5, 3)); b = RNG.standard_normal(6)
        ref = torch.nn.functional.conv1d(torch.tensor(x)[None], torch.tensor(w), torch.tensor(b),
                                         stride=stride, padding=1)[0].numpy()
        np.testing.assert_allclose(O.conv1d(x, w, b, stride), ref, atol=1e-12)


def test_conv_stem_identity_kernels():
    """Centre-tap identity kernels, zero bias: stem = GELU(GELU(x[:, 2j])) + PE[j]."""
    c, t, length = 8, 13, 9
    x = RNG.standard_normal((c, t))
    eye = np.zeros((c, c, 3)); eye[np.arange(c), np.arange(c), 1] = 1.0
    w = {"conv1_w": eye, "conv1_b": np.zeros(c), "conv2_w": eye, "conv2_b": np.zeros(c)}
    y = O.conv_stem(x, length, w)
    xm = x.copy(); xm[:, length:] = 0
    expect = O.gelu(O.gelu(xm[:, ::2])).T + O.sinusoids(O.encoder_positions(t), c)
    np.testing.assert_allclose(y, expect, atol=1e-14)


# ---------------------------------------------------------------- position
def test_sinusoid_closed_forms():
    d = 1280
    pe = O.sinusoids(1500, d)
    np.testing.assert_array_equal(pe[0, : d // 2], 0.0)
    np.testing.assert_array_equal(pe[0, d // 2:], 1.0)
    j = np.arange(1500)
    np.testing.assert_allclose(pe[:, 0], np.sin(j), atol=1e-12)                 # timescale 1
    np.testing.assert_allclose(pe[:, d // 2 - 1], np.sin(j * 1e-4), atol=1e-15)  # timescale 10000
    np.testing.assert_allclose(pe[:, d // 2], np.cos(j), atol=1e-12)
    np.testing.assert_allclose(pe[:, : d // 2] ** 2 + pe[:, d // 2:] ** 2, 1.0, atol=1e-12)
    # geometric spacing of the frequencies: ratio 10000^(-1/(d/2-1)) between neighbours
    small = O.sinusoids(2, 8)
    freqs = np.arcsin(small[1, :4])
    np.testing.assert_allclose(freqs[1:] / freqs[:-1], 10000.0 ** (-1.0 / 3.0), rtol=1e-12)


# ------------------------------------------------------------ elementwise
def test_gelu_pins():
    assert O.gelu(np.array([0.0]))[0] == 0.0
    x = np.linspace(-8, 8, 10001)
    np.testing.assert_allclose(O.gelu(x) - O.gelu(-x), x, atol=1e-13)
    ref = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in x])
    np.testing.assert_allclose(O.gelu(x), ref, atol=1e-15, rtol=1e-14)
    tref = torch.nn.functional.gelu(torch.tensor(x), approximate="none").numpy()
    np.testing.assert_allclose(O.gelu(x), tref, atol=1e-15, rtol=1e-13)
    np.testing.assert_allclose(O.gelu(np.array([1.0]))[0], 0.8413447460685429, rtol=1e-15)  # Phi(1)


def test_layer_norm_pins():
    x = RNG.standard_normal((7, 1280)) * 3 + 2
    y = O.layer_norm(x, np.ones(1280), np.zeros(1280), 1e-5)
    assert np.abs(y.mean(axis=1)).max() < 1e-6
    var = x.var(axis=1)
    np.testing.assert_allclose(y.var(axis=1), 1 - 1e-5 / (var + 1e-5), rtol=1e-12)
    g = RNG.standard_normal(1280); b = RNG.standard_normal(1280)
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (1280,), torch.tensor(g), torch.tensor(b), 1e-5)
    np.testing.assert_allclose(O.layer_norm(x, g, b, 1e-5), ref.numpy(), atol=1e-12)


# --------------------------------------------------------------- attention
def _attn_brute(q, k, v, n_heads, n_valid):
    s, hd = q.shape[0], q.shape[1] // n_heads
    out = np.zeros_like(q)
    for h in range(n_heads):
        for i in range(s):
            sc = [sum(q[i, h * hd + e] * k[j, h * hd + e] for e in range(hd)) / math.sqrt(hd)
                  for j in range(n_valid)]
            m = max(sc)
            p = [math.exp(z - m) for z in sc]
            tot = sum(p)
            for e in range(hd):
                out[i, h * hd + e] = sum(p[j] / tot * v[j, h * hd + e] for j in range(n_valid))
    return out


@pytest.mark.parametrize("s,n_valid,heads", [(1, 1, 1), (5, 3, 2), (8, 8, 2)])
def test_attention_bruteforce(s, n_valid, heads):
    hd = 4
    q, k, v = (RNG.standard_normal((s, heads * hd)) * 2 for _ in range(3))
    np.testing.assert_allclose(O.attention(q, k, v, heads, n_valid, hd), _attn_brute(q, k, v, heads, n_valid),
                               atol=1e-13)


def test_attention_invariants():
    s, heads, hd, n_valid = 12, 2, 64, 9
    q, k, v = (RNG.standard_normal((s, heads * hd)) for _ in range(3))
    # probabilities sum to 1: values of all ones give ones
    np.testing.assert_allclose(O.attention(q, k, np.ones_like(v), heads, n_valid), 1.0, atol=1e-14)
    base = O.attention(q, k, v, heads, n_valid)
    # masked keys/values do not matter at all
    k2, v2 = k.copy(), v.copy()
    k2[n_valid:] = 1e3; v2[n_valid:] = -7
    np.testing.assert_array_equal(O.attention(q, k2, v2, heads, n_valid), base)
    # permuting the valid keys (with their values) changes nothing (bidirectional, no positions)
    perm = np.concatenate([RNG.permutation(n_valid), np.arange(n_valid, s)])
    np.testing.assert_allclose(O.attention(q, k[perm], v[perm], heads, n_valid), base, atol=1e-14)
    # one query row alone gives the same row (rows are independent)
    np.testing.assert_allclose(O.attention(q[3:4], k, v, heads, n_valid), base[3:4], atol=1e-15)


def test_attention_matches_sdpa():
    s, heads, hd, n_valid = 10, 3, 64, 7
    q, k, v = (RNG.standard_normal((s, heads * hd)) for _ in range(3))
    t = lambda a: torch.tensor(a).reshape(s, heads, hd).transpose(0, 1)[None]
    mask = torch.zeros(s, s, dtype=torch.bool); mask[:, :n_valid] = True
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask)
    ref = ref[0].transpose(0, 1).reshape(s, heads * hd).numpy()
    np.testing.assert_allclose(O.attention(q, k, v, heads, n_valid), ref, atol=1e-13)


# ------------------------------------------------------------ whole blocks
def _rand_weights(d, m, f, layers, proj=None, std=0.2):
    w = {"conv1_w": RNG.standard_normal((d, m, 3)) * std, "conv1_b": RNG.standard_normal(d) * std,
         "conv2_w": RNG.standard_normal((d, d, 3)) * std, "conv2_b": RNG.standard_normal(d) * std,
         "lnpost_g": 1 + RNG.standard_normal(d) * std, "lnpost_b": RNG.standard_normal(d) * std}
    for l in range(layers):
        p = f"layers.{l}."
        for nm, shp in [("ln1_g", (d,)), ("ln1_b", (d,)), ("q_w", (d, d)), ("q_b", (d,)), ("k_w", (d, d)),
                        ("v_w", (d, d)), ("v_b", (d,)), ("o_w", (d, d)), ("o_b", (d,)), ("ln2_g", (d,)),
                        ("ln2_b", (d,)), ("fc1_w", (f, d)), ("fc1_b", (f,)), ("fc2_w", (d, f)), ("fc2_b", (d,))]:
            w[p + nm] = RNG.standard_normal(shp) * std + (1.0 if nm.endswith("_g") else 0.0)
    if proj:
        ph, po = proj
        w.update({"proj1_w": RNG.standard_normal((ph, d)) * std, "proj1_b": RNG.standard_normal(ph) * std,
                  "proj2_w": RNG.standard_normal((po, ph)) * std, "proj2_b": RNG.standard_normal(po) * std})
    return w


def _torch_tower(w, mel, length, d, heads, layers, pool, proj, chunk=0):
    """Independent composition from torch.nn layers (float64); chunk > 0 adds a
    block-diagonal attention mask (positions attend within their own chunk)."""
    T = lambda a: torch.tensor(np.asarray(a, np.float64))
    m, t = mel.shape
    c1 = torch.nn.Conv1d(m, d, 3, padding=1); c2 = torch.nn.Conv1d(d, d, 3, stride=2, padding=1)
    with torch.no_grad():
        c1.weight.copy_(T(w["conv1_w"])); c1.bias.copy_(T(w["conv1_b"]))
        c2.weight.copy_(T(w["conv2_w"])); c2.bias.copy_(T(w["conv2_b"]))
    x = T(mel).clone(); x[:, length:] = 0
    h = torch.nn.functional.gelu(c2(torch.nn.functional.gelu(c1(x[None]))))[0].T     # [P, d]
    h = h + T(O.sinusoids(h.shape[0], d))
    p = h.shape[0]
    n = -(-length // 2)
    enc = []
    for l in range(layers):
        lay = torch.nn.TransformerEncoderLayer(d, heads, w[f"layers.{l}.fc1_w"].shape[0], dropout=0.0,
                                               activation="gelu", batch_first=True, norm_first=True)
        pfx = f"layers.{l}."
        with torch.no_grad():
            lay.self_attn.in_proj_weight.copy_(torch.cat([T(w[pfx + "q_w"]), T(w[pfx + "k_w"]), T(w[pfx + "v_w"])]))
            lay.self_attn.in_proj_bias.copy_(torch.cat([T(w[pfx + "q_b"]), torch.zeros(d), T(w[pfx + "v_b"])]))
            lay.self_attn.out_proj.weight.copy_(T(w[pfx + "o_w"])); lay.self_attn.out_proj.bias.copy_(T(w[pfx + "o_b"]))
            lay.norm1.weight.copy_(T(w[pfx + "ln1_g"])); lay.norm1.bias.copy_(T(w[pfx + "ln1_b"]))
            lay.norm2.weight.copy_(T(w[pfx + "ln2_g"])); lay.norm2.bias.copy_(T(w[pfx + "ln2_b"]))
            lay.linear1.weight.copy_(T(w[pfx + "fc1_w"])); lay.linear1.bias.copy_(T(w[pfx + "fc1_b"]))
            lay.linear2.weight.copy_(T(w[pfx + "fc2_w"])); lay.linear2.bias.copy_(T(w[pfx + "fc2_b"]))
        lay.eval()
        enc.append(lay)
    pad = torch.zeros(1, p, dtype=torch.bool); pad[0, n:] = True
    blocks = None
    y = h[None]
    if chunk:
        # the valid rows alone (a padded query whose chunk holds no valid key would
        # give NaN, and NaN values reach valid rows through zero probabilities)
        y, pad = h[None, :n], None
        idx = torch.arange(n) // chunk
        blocks = idx[:, None] != idx[None, :]           # True: not allowed to attend
    with torch.no_grad():
        for lay in enc:
            y = lay(y, src_mask=blocks, src_key_padding_mask=pad)
        y = torch.nn.functional.layer_norm(y, (d,), T(w["lnpost_g"]), T(w["lnpost_b"]), 1e-5)[0]
        y = y[:n]
        if pool > 1:
            y = torch.nn.functional.avg_pool1d(y.T[None], pool, pool)[0].T
        if proj:
            y = torch.nn.functional.linear(torch.nn.functional.gelu(
                torch.nn.functional.linear(y, T(w["proj1_w"]), T(w["proj1_b"]))), T(w["proj2_w"]), T(w["proj2_b"]))
    return y.numpy()


@pytest.mark.parametrize("t,length,pool,proj,chunk", [
    (37, 37, 1, None, 0), (37, 23, 1, None, 0), (40, 40, 2, None, 0), (41, 30, 2, None, 0),
    (36, 36, 1, (48, 40), 0), (29, 17, 2, (48, 40), 0), (48, 48, 4, None, 0), (45, 29, 4, None, 0),
    (43, 40, 4, (48, 40), 0),
    (49, 49, 1, None, 7), (47, 33, 2, None, 5), (40, 31, 1, (48, 40), 6)])   # block-local attention
def test_tower_matches_torch_layers(t, length, pool, proj, chunk):
    d, m, f, heads, layers = 128, 8, 256, 2, 2
    w = _rand_weights(d, m, f, layers, proj)
    mel = RNG.uniform(-1.5, 1.5, (m, t))
    geo = Geo(layers, heads, pool, *(proj or (0, 0)), attn_chunk=chunk)
    got = O.encode_clip(geo, w, mel, length)
    ref = _torch_tower(w, mel, length, d, heads, layers, pool, proj, chunk)
    nv = O.valid_output_rows(geo, length)
    assert got.shape[0] == O.pooled_positions(O.encoder_positions(t), pool)
    assert nv == ref.shape[0]
    np.testing.assert_allclose(got[:nv], ref, atol=1e-10, rtol=1e-10)
    np.testing.assert_array_equal(got[nv:], 0.0)


def test_frame_mask_invariance():
    d, m, f, heads, layers = 128, 8, 256, 2, 1
    w = _rand_weights(d, m, f, layers)
    geo = Geo(layers, heads)
    mel = RNG.uniform(-1.5, 1.5, (m, 50))
    base = O.encode_clip(geo, w, mel, 31)
    mel2 = mel.copy(); mel2[:, 31:] = RNG.uniform(-9, 9, (m, 19))
    np.testing.assert_array_equal(O.encode_clip(geo, w, mel2, 31), base)
    # and a full-length clip is not affected by the mask at all
    np.testing.assert_array_equal(O.encode_clip(geo, w, mel, 50)[:25], O.encode_clip(geo, w, mel, 50)[:25])


def test_layer_limit_and_zero_layers():
    d, m, f, heads = 128, 8, 256, 2
    w = _rand_weights(d, m, f, 2)
    geo = Geo(2, heads)
    mel = RNG.uniform(-1.5, 1.5, (m, 20))
    y0 = O.encode_clip(geo, w, mel, 20, layers=0)
    stem = O.conv_stem(mel, 20, w)
    np.testing.assert_allclose(y0, O.layer_norm(stem, w["lnpost_g"], w["lnpost_b"]), atol=1e-14)


def test_chunked_attention_special_cases():
    """Block-local attention: a chunk covering the clip is full attention; a chunk of
    one position returns v itself (softmax over one key is 1); keys outside a
    chunk change nothing inside it."""
    s_len, heads = 23, 2
    q, k, v = (RNG.standard_normal((s_len, 64 * heads)) for _ in range(3))
    np.testing.assert_array_equal(O.chunked_attention(q, k, v, heads, 23), O.attention(q, k, v, heads))
    np.testing.assert_array_equal(O.chunked_attention(q, k, v, heads, 100), O.attention(q, k, v, heads))
    np.testing.assert_allclose(O.chunked_attention(q, k, v, heads, 1), v, rtol=0, atol=1e-15)
    k2, v2 = k.copy(), v.copy()
    k2[10:], v2[10:] = 7.0, -3.0                        # chunks of 5: rows 0..9 are chunks 0 and 1
    a = O.chunked_attention(q, k, v, heads, 5)
    b = O.chunked_attention(q, k2, v2, heads, 5)
    np.testing.assert_array_equal(a[:10], b[:10])
    assert not np.allclose(a[10:], b[10:])
