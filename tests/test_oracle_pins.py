"""Pins of the fp64 CPU oracle to things other than itself.

Each test checks the oracle against a closed form, an invariant the pages state,
brute force on tiny inputs, or an independent library implementation of the same
operation (numpy matmul, torch LayerNorm / GELU / SDPA / TransformerEncoderLayer,
HF transformers' AlbertModel).  Together they are chosen so that a dropped term,
a wrong sign, a transposed operand, a wrong head split, a causal mask or a
pre-LN/post-LN swap in the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

A = synth.ARCH


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- sizes ----

def test_parameter_counts_match_the_factorized_embedding_arithmetic():
    """Page 1, "1. Factorized embedding": tables 88,576; projection 98,304;
    total 186,880; unfactorized 531,456; savings 344,576 (~65%)."""
    s = synth.param_shapes()
    n = lambda k: int(np.prod(s[k]))
    assert n("word") == 22_784 and n("pos") == 65_536 and n("type") == 256
    tables = n("word") + n("pos") + n("type")
    assert tables == 88_576
    assert n("w_in") == 98_304
    assert tables + n("w_in") == 186_880
    unfact = A["vocab"] * A["hidden"] + A["max_pos"] * A["hidden"] + A["n_types"] * A["hidden"]
    assert unfact == 531_456
    assert unfact - 186_880 == 344_576
    assert round(100 * 344_576 / 531_456) == 65


def test_shared_layer_parameter_count():
    s = synth.param_shapes()
    layer = ["wq", "bq", "wk", "bk", "wv", "bv", "wo", "bo", "ln1_g", "ln1_b",
             "w1", "b1", "w2", "b2", "ln2_g", "ln2_b"]
    assert sum(int(np.prod(s[k])) for k in layer) == 5_513_984


# --------------------------------------------------------------- linear ----

def test_linear_matches_library_matmul_and_orientation():
    r = _rng(1)
    x, W, b = r.normal(size=(5, 7)), r.normal(size=(3, 7)), r.normal(size=3)
    y = oracle.linear(x, W, b)
    np.testing.assert_allclose(y, x @ W.T + b, rtol=1e-13, atol=1e-13)
    # W is [out, in]: output j only reads row j of W.
    W2 = W.copy()
    W2[1] += 1.0
    y2 = oracle.linear(x, W2, b)
    np.testing.assert_array_equal(y2[:, [0, 2]], y[:, [0, 2]])
    np.testing.assert_allclose(y2[:, 1] - y[:, 1], x.sum(1), rtol=1e-12)


def test_linear_is_exact_on_integers_and_keeps_the_small_term():
    # fp64 sum in ascending order keeps 1 in 1e8 + 1 - 1e8 (page 3, section A).
    x = np.array([[1e8, 1.0, -1e8]])
    W = np.ones((1, 3))
    assert oracle.linear(x, W, np.zeros(1))[0, 0] == 1.0


# ------------------------------------------------------------ LayerNorm ----

def test_layer_norm_zero_mean_unit_variance_closed_form():
    r = _rng(2)
    x = r.normal(3.0, 2.5, size=(6, 768))
    y = oracle.layer_norm(x, np.ones(768), np.zeros(768), 1e-12)
    assert np.all(np.abs(y.mean(1)) < 1e-12)
    var = x.var(1)
    np.testing.assert_allclose(y.var(1), var / (var + 1e-12), rtol=1e-12)


def test_layer_norm_eps_inside_the_sqrt():
    # a row with variance 1e-12 equal to eps: output scaled by 1/sqrt(2)
    x = np.array([[1e-6, -1e-6] * 64])
    y = oracle.layer_norm(x, np.ones(128), np.zeros(128), 1e-12)
    np.testing.assert_allclose(np.abs(y), 1 / math.sqrt(2), rtol=1e-9)


def test_layer_norm_constant_row_maps_to_beta_and_affine_order():
    r = _rng(3)
    g, b = r.normal(size=128), r.normal(size=128)
    y = oracle.layer_norm(np.full((1, 128), 4.25), g, b, 1e-12)
    np.testing.assert_array_equal(y[0], b)
    x = r.normal(size=(4, 128))
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (128,), torch.tensor(g),
                                         torch.tensor(b), eps=1e-12).numpy()
    np.testing.assert_allclose(oracle.layer_norm(x, g, b, 1e-12), ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- GELU ----

def test_gelu_closed_forms():
    assert oracle.gelu_scalar(0.0) == 0.0
    for x in (0.1, 0.7, 1.3, 2.9, 5.0):
        # GELU(x) - GELU(-x) = x holds exactly for the tanh form
        assert abs(oracle.gelu_scalar(x) - oracle.gelu_scalar(-x) - x) < 1e-15
    assert abs(oracle.gelu_scalar(30.0) - 30.0) < 1e-12
    assert abs(oracle.gelu_scalar(-30.0)) < 1e-12
    # spot value from the formula in long form
    c = math.sqrt(2 / math.pi)
    assert abs(oracle.gelu_scalar(1.0) - 0.5 * (1 + math.tanh(c * 1.044715))) < 1e-15


def test_gelu_is_the_tanh_variant_not_erf():
    x = np.linspace(-6, 6, 2001)
    y = oracle.gelu(x)
    t = torch.tensor(x)
    tanh_ref = torch.nn.functional.gelu(t, approximate="tanh").numpy()
    erf_ref = torch.nn.functional.gelu(t).numpy()
    np.testing.assert_allclose(y, tanh_ref, rtol=1e-13, atol=1e-15)
    assert np.max(np.abs(y - erf_ref)) > 1e-4


# ------------------------------------------------------------ attention ----

def _long_form_attention(q, k, v, key_mask, heads):
    """Brute force: weights exp(s)/sum exp(s) without max subtraction, math.fsum."""
    T, D = q.shape
    dh = D // heads
    out = np.zeros((T, D))
    for h in range(heads):
        sl = slice(h * dh, (h + 1) * dh)
        for t in range(T):
            w = []
            for u in range(T):
                if key_mask[u]:
                    s = math.fsum(q[t, sl] * k[u, sl]) / math.sqrt(dh)
                    w.append((u, math.exp(s)))
            den = math.fsum(e for _, e in w)
            for i in range(dh):
                out[t, h * dh + i] = math.fsum(e * v[u, h * dh + i] for u, e in w) / den
    return out


@pytest.mark.parametrize("T,heads,dh", [(1, 1, 2), (2, 1, 3), (3, 2, 2), (4, 2, 4)])
def test_attention_brute_force_tiny(T, heads, dh):
    r = _rng(10 + T)
    q, k, v = (r.normal(size=(T, heads * dh)) for _ in range(3))
    for key_mask in ([1] * T, [1] * max(1, T - 1) + [0] * (T - max(1, T - 1))):
        key_mask = np.array(key_mask, np.uint8)
        got = oracle.attention(q, k, v, key_mask, heads)
        np.testing.assert_allclose(got, _long_form_attention(q, k, v, key_mask, heads),
                                   rtol=1e-12, atol=1e-13)


def test_attention_single_key_returns_its_value():
    r = _rng(4)
    q, k, v = (r.normal(size=(1, 768)) for _ in range(3))
    np.testing.assert_allclose(oracle.attention(q, k, v, np.ones(1, np.uint8), 12), v,
                               rtol=0, atol=1e-15)


def test_attention_identical_keys_returns_mean_of_valid_values():
    r = _rng(5)
    T = 9
    q = r.normal(size=(T, 768))
    k = np.tile(r.normal(size=(1, 768)), (T, 1))
    v = r.normal(size=(T, 768))
    key_mask = np.array([1] * 6 + [0] * 3, np.uint8)
    got = oracle.attention(q, k, v, key_mask, 12)
    np.testing.assert_allclose(got, np.tile(v[:6].mean(0), (T, 1)), rtol=1e-12, atol=1e-14)


def test_attention_matches_library_sdpa_with_key_padding_and_head_split():
    r = _rng(6)
    T, heads, dh = 11, 12, 64
    q, k, v = (r.normal(size=(T, heads * dh)) for _ in range(3))
    key_mask = np.array([1] * 8 + [0] * 3, np.uint8)
    got = oracle.attention(q, k, v, key_mask, heads)
    th = lambda a: torch.tensor(a).view(T, heads, dh).transpose(0, 1)  # [h, T, dh]
    am = torch.tensor(key_mask.astype(bool))[None, None, :].expand(heads, T, T)
    ref = torch.nn.functional.scaled_dot_product_attention(th(q), th(k), th(v), attn_mask=am)
    ref = ref.transpose(0, 1).reshape(T, heads * dh).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_attention_is_bidirectional():
    r = _rng(7)
    T = 6
    q, k, v = (r.normal(size=(T, 64)) for _ in range(3))
    m = np.ones(T, np.uint8)
    a = oracle.attention(q, k, v, m, 1)
    v2 = v.copy()
    v2[-1] += 1.0
    b = oracle.attention(q, k, v2, m, 1)
    assert np.all(np.abs(a[0] - b[0]) > 0)  # the first token sees the last one


# -------------------------------------------------------- whole encoder ----

def _hf_model(w, n_layers, n_groups=1):
    from transformers import AlbertConfig, AlbertModel
    cfg = AlbertConfig(vocab_size=A["vocab"], embedding_size=A["emb"], hidden_size=A["hidden"],
                       num_hidden_layers=n_layers, num_hidden_groups=n_groups,
                       num_attention_heads=A["heads"], intermediate_size=A["ffn"],
                       inner_group_num=1, hidden_act="gelu_new", hidden_dropout_prob=0.0,
                       attention_probs_dropout_prob=0.0, max_position_embeddings=A["max_pos"],
                       type_vocab_size=A["n_types"], layer_norm_eps=A["ln_eps"],
                       attn_implementation="eager")
    m = AlbertModel(cfg, add_pooling_layer=False).double().eval()
    shared = {
        "embeddings.word_embeddings.weight": "word",
        "embeddings.position_embeddings.weight": "pos",
        "embeddings.token_type_embeddings.weight": "type",
        "embeddings.LayerNorm.weight": "emb_ln_g", "embeddings.LayerNorm.bias": "emb_ln_b",
        "encoder.embedding_hidden_mapping_in.weight": "w_in",
        "encoder.embedding_hidden_mapping_in.bias": "b_in",
    }
    sd = m.state_dict()
    with torch.no_grad():
        for hf, ours in shared.items():
            sd[hf].copy_(torch.tensor(w[ours], dtype=torch.float64))
        for g in range(n_groups):
            lay = f"encoder.albert_layer_groups.{g}.albert_layers.0."
            for hf, ours in _layer_names(lay).items():
                src = w[ours][g] if n_groups > 1 else w[ours]
                sd[hf].copy_(torch.tensor(src, dtype=torch.float64))
    return m


def _layer_names(lay):
    return {
        lay + "attention.query.weight": "wq", lay + "attention.query.bias": "bq",
        lay + "attention.key.weight": "wk", lay + "attention.key.bias": "bk",
        lay + "attention.value.weight": "wv", lay + "attention.value.bias": "bv",
        lay + "attention.dense.weight": "wo", lay + "attention.dense.bias": "bo",
        lay + "attention.LayerNorm.weight": "ln1_g", lay + "attention.LayerNorm.bias": "ln1_b",
        lay + "ffn.weight": "w1", lay + "ffn.bias": "b1",
        lay + "ffn_output.weight": "w2", lay + "ffn_output.bias": "b2",
        lay + "full_layer_layer_norm.weight": "ln2_g", lay + "full_layer_layer_norm.bias": "ln2_b",
    }


@pytest.mark.parametrize("n_exec", [1, 12])
def test_encoder_matches_hf_albert_model(n_exec):
    """A library ALBERT (transformers' AlbertModel, fully shared layer, gelu_new,
    eps 1e-12) with the same parameters gives the same [T, 768] states."""
    w = synth.make_weights(seed=21, bf16=False, ln_affine="random")
    r = _rng(22)
    B, T = 3, 20
    L = [20, 13, 5]
    ids = np.zeros((B, T), np.int64)
    mask = np.zeros((B, T), np.uint8)
    for b in range(B):
        ids[b, 1:L[b] - 1] = r.integers(1, A["vocab"], L[b] - 2)
        ids[b, L[b]:] = r.integers(0, A["vocab"], T - L[b])  # arbitrary pad ids
        mask[b, :L[b]] = 1
    model = oracle.Model(w, A, n_exec=n_exec, out_dim=0)
    got = model.encode(ids, mask)
    hf = _hf_model(w, n_exec)
    with torch.no_grad():
        ref = hf(input_ids=torch.tensor(ids), attention_mask=torch.tensor(mask.astype(np.int64)),
                 token_type_ids=torch.zeros_like(torch.tensor(ids))).last_hidden_state.numpy()
    for b in range(B):
        np.testing.assert_allclose(got[b, :L[b]], ref[b, :L[b]], rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("n_groups", [2, 3, 12])
def test_grouped_sharing_matches_hf_albert_model(n_groups):
    """Grouped sharing (n_groups weight sets over 12 executions) against
    transformers' AlbertModel with num_hidden_groups = n_groups."""
    w = synth.make_weights(seed=23, bf16=False, ln_affine="random", n_groups=n_groups)
    r = _rng(24)
    T, L = 18, 15
    ids = np.zeros(T, np.int64)
    ids[1:L - 1] = r.integers(1, A["vocab"], L - 2)
    mask = np.array([1] * L + [0] * (T - L), np.uint8)
    got = oracle.encode_grouped(w, A, ids, mask, n_groups, n_exec=12, out_dim=0)
    hf = _hf_model(w, 12, n_groups)
    with torch.no_grad():
        ref = hf(input_ids=torch.tensor(ids[None]), attention_mask=torch.tensor(mask[None].astype(np.int64)),
                 token_type_ids=torch.zeros(1, T, dtype=torch.int64)).last_hidden_state.numpy()[0]
    np.testing.assert_allclose(got[:L], ref[:L], rtol=1e-9, atol=1e-9)
    assert np.all(got[L:] == 0)


def test_grouped_sharing_with_one_group_is_the_shared_model():
    w = synth.make_weights(seed=25, bf16=False, ln_affine="random")
    r = _rng(26)
    ids = np.zeros(12, np.int64)
    ids[1:9] = r.integers(1, A["vocab"], 8)
    mask = np.array([1] * 10 + [0] * 2, np.uint8)
    a = oracle.encode_grouped(w, A, ids, mask, 1)
    b = oracle.Model(w, A).encode(ids, mask)
    np.testing.assert_allclose(a[:10], b[:10], rtol=1e-12, atol=1e-12)


def test_one_layer_matches_library_post_ln_transformer_layer():
    w = synth.make_weights(seed=31, bf16=False, ln_affine="random")
    r = _rng(32)
    T, L = 17, 12
    x = r.normal(size=(T, 768))
    mask = np.array([1] * L + [0] * (T - L), np.uint8)
    got = oracle.Model(w, A).layer(x, mask)
    lay = torch.nn.TransformerEncoderLayer(
        768, 12, dim_feedforward=2048, dropout=0.0,
        activation=lambda t: torch.nn.functional.gelu(t, approximate="tanh"),
        layer_norm_eps=1e-12, batch_first=True, norm_first=False).double().eval()
    with torch.no_grad():
        lay.self_attn.in_proj_weight.copy_(torch.tensor(np.concatenate([w["wq"], w["wk"], w["wv"]])))
        lay.self_attn.in_proj_bias.copy_(torch.tensor(np.concatenate([w["bq"], w["bk"], w["bv"]])))
        lay.self_attn.out_proj.weight.copy_(torch.tensor(w["wo"]))
        lay.self_attn.out_proj.bias.copy_(torch.tensor(w["bo"]))
        lay.linear1.weight.copy_(torch.tensor(w["w1"]))
        lay.linear1.bias.copy_(torch.tensor(w["b1"]))
        lay.linear2.weight.copy_(torch.tensor(w["w2"]))
        lay.linear2.bias.copy_(torch.tensor(w["b2"]))
        lay.norm1.weight.copy_(torch.tensor(w["ln1_g"]))
        lay.norm1.bias.copy_(torch.tensor(w["ln1_b"]))
        lay.norm2.weight.copy_(torch.tensor(w["ln2_g"]))
        lay.norm2.bias.copy_(torch.tensor(w["ln2_b"]))
        ref = lay(torch.tensor(x)[None], src_key_padding_mask=torch.tensor(mask == 0)[None])[0]
    np.testing.assert_allclose(got[:L], ref.numpy()[:L], rtol=1e-10, atol=1e-10)


def test_final_projection_matches_library_linear():
    w = synth.make_weights(seed=41, bf16=True)
    ids, mask, L = synth.make_batch(synth.Workload("t", 2, 9, "uniform", lo=3, hi=9, seed=5))
    full = oracle.Model(w, A, n_exec=2, out_dim=512).encode(ids, mask)
    hid = oracle.Model(w, A, n_exec=2, out_dim=0).encode(ids, mask)
    ref = torch.nn.functional.linear(torch.tensor(hid), torch.tensor(w["w_out"], dtype=torch.float64),
                                     torch.tensor(w["b_out"], dtype=torch.float64)).numpy()
    np.testing.assert_allclose(full, ref, rtol=1e-12, atol=1e-12)


def test_padding_invariance():
    """Valid outputs do not change when the sequence is padded with any ids."""
    w = synth.make_weights(seed=51, bf16=True)
    r = _rng(52)
    L, T = 10, 23
    ids = np.zeros(L, np.int64)
    ids[1:-1] = r.integers(1, A["vocab"], L - 2)
    m = oracle.Model(w, A, n_exec=3)
    base = m.encode(ids, np.ones(L, np.uint8))
    for trial in range(2):
        pid = np.concatenate([ids, r.integers(0, A["vocab"], T - L)])
        pm = np.array([1] * L + [0] * (T - L), np.uint8)
        np.testing.assert_array_equal(m.encode(pid, pm)[:L], base)


def test_n_exec_is_the_fold_of_one_shared_layer():
    w = synth.make_weights(seed=61, bf16=True)
    ids, mask, L = synth.make_batch(synth.Workload("t", 1, 12, "full", seed=3))
    ids, mask = ids[0], mask[0]
    m0 = oracle.Model(w, A, n_exec=0, out_dim=0)
    x = m0.encode(ids, mask)
    np.testing.assert_allclose(x, oracle.linear(m0.embed(ids, mask), w["w_in"], w["b_in"]),
                               rtol=0, atol=0)
    m12 = oracle.Model(w, A, n_exec=12, out_dim=0)
    for _ in range(12):
        x = m12.layer(x, mask)
    np.testing.assert_array_equal(m12.encode(ids, mask), x)


def test_permutation_equivariance_without_positions():
    """With the position table zeroed the encoder is permutation-equivariant; a
    causal or shifted mask would break this."""
    w = synth.make_weights(seed=71, bf16=False)
    w["pos"] = np.zeros_like(w["pos"])
    r = _rng(72)
    T = 8
    ids = r.integers(0, A["vocab"], T)
    perm = r.permutation(T)
    m = oracle.Model(w, A, n_exec=2)
    a = m.encode(ids, np.ones(T, np.uint8))
    b = m.encode(ids[perm], np.ones(T, np.uint8))
    np.testing.assert_allclose(b, a[perm], rtol=1e-10, atol=1e-12)


def test_embedding_is_three_table_sum_then_layer_norm():
    w = synth.make_weights(seed=81, bf16=False, ln_affine="random")
    ids = np.array([0, 5, 177, 3, 0], np.int64)
    m = oracle.Model(w, A)
    e = m.embed(ids, np.ones(5, np.uint8))
    s = torch.tensor(w["word"][ids] + w["pos"][:5] + w["type"][0], dtype=torch.float64)
    ref = torch.nn.functional.layer_norm(s, (128,), torch.tensor(w["emb_ln_g"], dtype=torch.float64),
                                         torch.tensor(w["emb_ln_b"], dtype=torch.float64), eps=1e-12)
    np.testing.assert_allclose(e, ref.numpy(), rtol=1e-6, atol=1e-6)


def test_oracle_rejects_out_of_range_ids():
    w = synth.make_weights(seed=91, bf16=True)
    m = oracle.Model(w, A, n_exec=1)
    with pytest.raises(ValueError):
        m.encode(np.array([0, 178, 0]), np.ones(3, np.uint8))
    with pytest.raises(ValueError):
        m.encode(np.array([0, -1, 0]), np.ones(3, np.uint8))
