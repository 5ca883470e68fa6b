"""Pins of the CPU oracle against facts that do not come from the oracle itself:
format tables of the OCP specs, hand-worked examples (tests/golden), library
routines (ml_dtypes, torch), brute force on tiny inputs, closed forms and the
invariants the glm5next_mlp docs state in "Traps this module exists to hold".
"""
import itertools
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from conftest import golden_comment_field, golden_lines
from oracle import formats as F
from oracle import site as S
from routed_nvfp4_expert_b200 import synthetic as syn


# ------------------------------------------------------------------ formats

def test_e2m1_table_matches_ocp_spec():
    for code, val in golden_lines("e2m1_table.txt"):
        v = F.e2m1_value(int(code))
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val)), code


def test_e2m1_table_matches_ml_dtypes():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(F.e2m1_value(np.arange(16)), lib)
    assert np.array_equal(np.signbit(F.e2m1_value(np.arange(16))), np.signbit(lib))


def test_e4m3_points_match_ofp8_spec():
    for hx, val in golden_lines("e4m3_points.txt"):
        v = float(F.e4m3_value(int(hx, 16)))
        if val == "nan":
            assert math.isnan(v), hx
        else:
            assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val)), hx


def test_e4m3_exhaustive_matches_torch_and_ml_dtypes():
    b = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_value(b)
    t = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    m = b.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for lib in (t, m):
        assert np.array_equal(np.isnan(ours), np.isnan(lib))
        ok = ~np.isnan(ours)
        assert np.array_equal(ours[ok], lib[ok])
        assert np.array_equal(np.signbit(ours[ok]), np.signbit(lib[ok]))


def test_bf16_widen_and_round_match_torch():
    rng = np.random.default_rng(5)
    f = (rng.standard_normal(20000) * 10 ** rng.uniform(-30, 30, 20000)).astype(np.float32)
    # exact midpoints between neighbouring bf16 values: low 16 bits = 0x8000
    mid = (rng.integers(0, 2 ** 16, 5000, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32).view(np.float32)
    mid = mid[np.isfinite(mid)]
    f = np.concatenate([f, mid, np.float32([0.0, -0.0, 1.0, -1.0])])
    ref = torch.from_numpy(f).to(torch.bfloat16)
    ours = F.f32_to_bf16_bits(f)
    assert np.array_equal(ours, ref.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(F.bf16_value(ours), ref.to(torch.float64).numpy())


def test_e2m1_encoder_ties_hand_table():
    for val, code in golden_lines("e2m1_ties.txt"):
        assert int(F.e2m1_encode_satfinite(np.float32(val))) == int(code, 16), val


def test_e2m1_encoder_matches_ml_dtypes_on_all_midpoints_and_randoms():
    grid = F.e2m1_value(np.arange(8))
    mids = (grid[:-1] + grid[1:]) / 2
    probes = np.concatenate([mids, np.nextafter(mids.astype(np.float32), 0), np.nextafter(mids.astype(np.float32), 10),
                             grid, np.random.default_rng(1).uniform(0, 8, 20000)]).astype(np.float32)
    probes = np.concatenate([probes, -probes])
    lib = probes.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(F.e2m1_encode_satfinite(probes), lib)


def test_e4m3_encoder_matches_ml_dtypes_below_overflow():
    grid = F.e4m3_value(np.arange(0x7F))
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    rng = np.random.default_rng(2)
    rnd = (2.0 ** rng.uniform(-12, 8.8, 50000)).astype(np.float32)
    probes = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 1000), grid.astype(np.float32), rnd])
    probes = probes[probes < 464]
    probes = np.concatenate([probes, -probes])
    lib = probes.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(F.e4m3_encode_satfinite(probes), lib)
    # satfinite: anything finite above the largest value becomes 448
    assert list(F.e4m3_encode_satfinite(np.float32([464, 500, 1e30, -1e30]))) == [0x7E, 0x7E, 0x7E, 0xFE]


def test_dequant_hand_worked_dot_product():
    g = {ln[0]: ln[1:] for ln in golden_lines("dequant_dot.txt")}
    packed = np.array([int(h, 16) for h in g["packed"]], np.uint8)[None, :]
    scales = np.array([int(g["scale"][0], 16)], np.uint8)[None, :]
    w = F.nvfp4_dequant(packed, scales, np.float32(g["tensor_scale"][0]))
    x = np.array([float(v) for v in g["x"]])
    assert float(w[0] @ x) == float(g["dot"][0])


def test_dequant_matches_ml_dtypes_on_random_bank():
    codes, scales, ts = syn.nvfp4_bank(3, "gate", 2, 8, 64, 0.02)
    for e in range(2):
        lo = (codes[e] & 0xF).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        hi = (codes[e] >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        v = np.empty((8, 64))
        v[:, 0::2], v[:, 1::2] = lo, hi
        s = np.repeat(scales[e].view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=1)
        assert np.array_equal(F.nvfp4_dequant(codes[e], scales[e], ts[e]), v * s * float(ts[e]))


def test_act_quant_hand_worked_example():
    rows = golden_lines("act_quant_example.txt")
    a = np.array([[float(r[0]) for r in rows]], np.float32)
    want_codes = np.array([int(r[2], 16) for r in rows], np.uint8)
    c, s, t = F.quantize_rows_nvfp4(a)
    assert np.array_equal(F.unpack_nibbles(c)[0], want_codes)
    assert [int(v) for v in s[0]] == [int(h, 16) for h in golden_comment_field("act_quant_example.txt", "scales_hex")]
    assert t.view(np.uint32)[0] == int(golden_comment_field("act_quant_example.txt", "tsx_hex")[0], 16)


def test_act_quant_dequant_hand_worked_example():
    """dequant_rows_nvfp4 on the hand-worked row: every element equals code
    value x e4m3(scale) x tsx as worked out by hand, sign of zero included."""
    rows = golden_lines("act_quant_example.txt")
    a = np.array([[float(r[0]) for r in rows]], np.float32)
    c, s, t = F.quantize_rows_nvfp4(a)
    got = F.dequant_rows_nvfp4(c, s, t)[0]
    want = golden_lines("act_quant_dequant.txt")
    assert [int(w[0], 16) for w in want] == list(F.unpack_nibbles(c)[0])
    for g, (_, v) in zip(got, want):
        assert g == float(v) and math.copysign(1, g) == math.copysign(1, float(v)), (g, v)
    # per-block scale broadcast: the same codes under swapped block scales
    # decode block 0 with 0x59 and block 1 with 0x7E
    got2 = F.dequant_rows_nvfp4(c, s[:, ::-1].copy(), t)[0]
    assert got2[0] == 6 * 18 * 2.0 ** -9 and got2[16] == 6 * 448 * 2.0 ** -9
    # the row scale multiplies every element: twice tsx, twice the values
    got3 = F.dequant_rows_nvfp4(c, s, (t * 2).astype(np.float32))[0]
    assert np.array_equal(got3, 2 * got)


def test_router_logits_hand_worked_example():
    """l = Wr . x on a non-square router (E = 3, H = 5), worked by hand."""
    rows = golden_lines("router_logits_example.txt")
    x = np.array([[float(v) for v in r[1:]] for r in rows if r[0] == "x"], np.float32)
    w = np.array([[float(v) for v in r[1:]] for r in rows if r[0] == "w"], np.float32)
    want = np.array([[float(v) for v in r[1:]] for r in rows if r[0] == "logits"])
    got = S.router_logits(F.f32_to_bf16_bits(x), w)
    assert got.shape == (2, 3)
    assert np.array_equal(got, want)


def test_act_quant_matches_ml_dtypes_steps():
    """The same steps with the two roundings done by ml_dtypes."""
    rng = np.random.default_rng(7)
    a = F.bf16_value(syn._to_bf16_bits(rng.standard_normal((64, 256)) * 10 ** rng.uniform(-3, 3, (64, 1))))
    a = a.astype(np.float32)
    a[3] = 0.0                      # zero row
    a[5, 16:32] = 0.0               # zero block
    c, s, t = F.quantize_rows_nvfp4(a)
    r = np.abs(a).max(axis=1)
    tsx = r / np.float32(2688.0)
    assert np.array_equal(t, tsx)
    amax = np.abs(a).reshape(64, 16, 16).max(axis=2)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (amax / np.float32(6)) / tsx[:, None]
    q = np.nan_to_num(q, nan=0.0)
    sb = np.minimum(q, np.float32(448)).astype(ml_dtypes.float8_e4m3fn)
    assert np.array_equal(s, sb.view(np.uint8))
    d = sb.astype(np.float32) * tsx[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = a.reshape(64, 16, 16) / d[:, :, None]
    ratio = np.where(d[:, :, None] == 0, np.float32(0), ratio).astype(np.float32)
    codes = ratio.astype(ml_dtypes.float4_e2m1fn).view(np.uint8).reshape(64, 256) & 0xF
    assert np.array_equal(F.unpack_nibbles(c), codes)
    # the zero row encodes to all-zero bytes
    assert not c[3].any() and not s[3].any() and t[3] == 0


# ------------------------------------------------------------------ router

def test_sigmoid_matches_torch():
    l = np.random.default_rng(3).standard_normal(10000).astype(np.float32) * 8
    l = np.concatenate([l, np.float32([0, -100, 100, -1e30, 1e30])])
    ref = torch.sigmoid(torch.from_numpy(l).double()).float().numpy()
    assert np.array_equal(S.sigmoid_f32(l), ref)
    assert S.sigmoid_f32(np.float32([0.0]))[0] == np.float32(0.5)


def _valid_topk_subset(key, k):
    """Brute force: the unique k-subset whose every member beats every
    non-member under (key descending, index ascending)."""
    E = key.size
    better = lambda a, b: key[a] > key[b] or (key[a] == key[b] and a < b)
    found = [c for c in itertools.combinations(range(E), k)
             if all(better(i, j) for i in c for j in range(E) if j not in c)]
    assert len(found) == 1
    return set(found[0])


@pytest.mark.parametrize("ties", [False, True])
def test_topk_brute_force_all_subsets(ties):
    rng = np.random.default_rng(11 + ties)
    E, k, T = 16, 4, 12
    if ties:   # few distinct values -> many exactly equal keys
        logits = rng.choice(np.float32([0.0, 1.0, -1.0]), (T, E))
        bias = rng.choice(np.float32([0.0, 0.5]), E)
    else:
        logits = rng.standard_normal((T, E)).astype(np.float32)
        bias = (rng.standard_normal(E) * 0.5).astype(np.float32)
    ids = S.select_experts(logits, bias, k)
    key = S.selection_keys(logits, bias)
    for t in range(T):
        assert set(ids[t].tolist()) == _valid_topk_subset(key[t], k)
        kk = key[t, ids[t]]
        for a, b in zip(ids[t][:-1], ids[t][1:]):   # rank order
            assert key[t, a] > key[t, b] or (key[t, a] == key[t, b] and a < b)
        assert kk.dtype == np.float32


def test_k1_weight_is_rsf_exactly():
    rng = np.random.default_rng(4)
    l64 = rng.standard_normal((50, 16))
    ids = S.select_experts(l64.astype(np.float32), np.zeros(16, np.float32), 1)
    w = S.routing_weights(l64, ids, 2.5)
    assert np.all(w == 2.5)


def test_weights_renormalise_to_rsf_and_ignore_bias():
    rng = np.random.default_rng(9)
    l64 = rng.standard_normal((40, 32))
    b1 = (rng.standard_normal(32) * 0.5).astype(np.float32)
    ids1 = S.select_experts(l64.astype(np.float32), b1, 8)
    ids0 = S.select_experts(l64.astype(np.float32), np.zeros(32, np.float32), 8)
    assert not np.array_equal(ids0, ids1)            # the bias changes selection
    w1 = S.routing_weights(l64, ids1, 2.5)
    assert np.allclose(w1.sum(axis=1), 2.5, rtol=0, atol=1e-12)
    # shifting every bias by a power of two keeps the order (exact fp32 adds
    # for these magnitudes) -> same ids -> bitwise the same weights
    b2 = (b1 + np.float32(4.0)).astype(np.float32)
    ids2 = S.select_experts(l64.astype(np.float32), b2, 8)
    if np.array_equal(ids1, ids2):
        assert np.array_equal(S.routing_weights(l64, ids2, 2.5), w1)
    # the emitted weight follows the unbiased score: the chosen expert with the
    # largest logit has the largest weight, whatever the bias did
    for t in range(40):
        j_best = np.argmax(l64[t, ids1[t]])
        assert np.argmax(w1[t]) == j_best


# ------------------------------------------------------------------ MLP and site

def _tiny(**kw):
    wl = syn.WORKLOADS["tiny_t4"]
    import dataclasses
    wl = dataclasses.replace(wl, **kw)
    inp = syn.make_site(wl, seed=0)
    cfg = S.SiteConfig(hidden=wl.H, intermediate=wl.I, shared_intermediate=wl.Is, num_experts=wl.E,
                       local_begin=0, local_end=wl.E, top_k=wl.k, routed_scaling_factor=wl.rsf,
                       swiglu_limit=wl.limit)
    return wl, inp, cfg


def test_clamped_swiglu_asymmetric_closed_form():
    L = 7.0
    g = np.array([10.0, 10.0, -10.0, 1.0, 1.0, 0.0])
    u = np.array([10.0, -10.0, 3.0, 20.0, -20.0, 5.0])
    h = S.clamped_swiglu(g, u, L)
    silu = lambda z: z / (1 + math.exp(-z))
    want = [silu(7) * 7, silu(7) * -7, silu(-10) * 3, silu(1) * 7, silu(1) * -7, 0.0]
    assert np.allclose(h, want, rtol=1e-15, atol=0)
    # the gate is NOT bounded below: g = -10 passes through unclamped
    assert h[2] == silu(-10) * 3


def test_textbook_reduction_single_expert_matches_torch():
    """E = k = 1, rsf = 1, no shared expert, L = inf: the site is a plain SwiGLU
    MLP on the dequantised weights (dequantised here with ml_dtypes)."""
    wl, inp, cfg = _tiny(E=1, k=1, Is=0, rsf=1.0, limit=math.inf)
    cfg.top_k, cfg.num_experts, cfg.local_end = 1, 1, 1
    out = S.site_forward(inp, cfg, "decode")

    def deq(p):
        c, s, t = inp[f"{p}_codes"][0], inp[f"{p}_scales"][0], float(inp[f"{p}_ts"][0])
        v = np.empty((c.shape[0], c.shape[1] * 2))
        v[:, 0::2] = (c & 0xF).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        v[:, 1::2] = (c >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        return torch.from_numpy(v * np.repeat(s.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, 1) * t)

    x = torch.from_numpy(inp["x"].view(np.int16).copy()).view(torch.bfloat16).double()
    wg, wu, wd = deq("gate"), deq("up"), deq("down")
    ref = torch.nn.functional.linear(torch.nn.functional.silu(torch.nn.functional.linear(x, wg))
                                     * torch.nn.functional.linear(x, wu), wd)
    assert np.allclose(out["y"], ref.numpy(), rtol=1e-12, atol=1e-15)


def test_zero_token_gives_zero_and_bias_only_selection():
    wl, inp, cfg = _tiny()
    inp["x"][2] = 0
    out = S.site_forward(inp, cfg, "decode")
    assert np.all(out["logits"][2] == 0.0)
    want = np.lexsort((np.arange(wl.E), -inp["router_bias"].astype(np.float64)))[:wl.k]
    assert np.array_equal(out["ids"][2], want)
    assert np.all(out["y"][2] == 0.0)
    assert np.allclose(out["weights"][2], wl.rsf / wl.k, rtol=0, atol=0)


def test_shared_expert_is_never_scaled():
    wl, inp, cfg = _tiny()
    outs = {}
    for rsf in (0.0, 2.5, 5.0):
        cfg.routed_scaling_factor = rsf
        outs[rsf] = S.site_forward(inp, cfg, "decode", want_parts=True)
    assert np.array_equal(outs[0.0]["y"], outs[0.0]["shared"])
    d1 = outs[5.0]["y"] - outs[2.5]["y"]
    d0 = outs[2.5]["y"] - outs[0.0]["y"]
    assert np.allclose(d1, d0, rtol=1e-12, atol=1e-15)
    assert np.abs(outs[2.5]["shared"]).max() > 0


def test_clamp_fires_only_on_tails():
    wl, inp, cfg = _tiny()
    base = S.site_forward(inp, cfg, "decode")
    assert base["clamp_fired"] == 0
    cfg.swiglu_limit = math.inf
    assert np.array_equal(S.site_forward(inp, cfg, "decode")["y"], base["y"])
    # tails: activations x 64 push pre-activations past L
    wl2, inp2, cfg2 = _tiny(x_scale=64.0)
    hot = S.site_forward(inp2, cfg2, "decode")
    assert 0 < hot["clamp_fired"] < hot["clamp_total"]
    cfg2.swiglu_limit = math.inf
    assert not np.allclose(S.site_forward(inp2, cfg2, "decode")["y"], hot["y"])


def test_stress_recipe_fires_the_clamp_on_about_five_percent():
    """The stress workload's x8 activations make the clamp fire on ~5% of the
    gate/up elements (the stress prefill config), while the plain prefill
    workload's never reach it (the clamp is invisible off the tails)."""
    from helpers import oracle_cfg, site_inputs, workload
    for name, lo, hi in (("stress_t16384", 0.03, 0.07), ("prefill_t4096", 0.0, 1e-4)):
        wl = workload(name)
        inp = site_inputs(wl)
        rng = np.random.default_rng(11)
        tokens = np.setdiff1d(rng.choice(wl.T, 40, replace=False), inp.get("tie_tokens", []))[:24]
        out = S.site_forward(inp, oracle_cfg(wl), "decode", tokens=tokens)
        frac = out["clamp_fired"] / out["clamp_total"]
        assert lo <= frac <= hi, (name, frac)


def test_local_range_masks_remote_experts():
    wl, inp, cfg = _tiny()
    full = S.site_forward(inp, cfg, "decode", want_parts=True)
    cfg.local_begin, cfg.local_end = 0, wl.E // 2
    lo = S.site_forward(inp, cfg, "decode", want_parts=True)
    cfg.local_begin, cfg.local_end = wl.E // 2, wl.E
    hi = S.site_forward(inp, cfg, "decode", want_parts=True)
    # same ids and weights on every "rank" (the router ranks the FULL count)
    assert np.array_equal(lo["ids"], full["ids"]) and np.array_equal(hi["ids"], full["ids"])
    # the two masked partials (shared counted once) add up to the full site
    assert np.allclose(lo["y"] + hi["y"] - full["shared"], full["y"], rtol=1e-12, atol=1e-15)


def test_stress_tie_tokens_pick_lowest_indices_of_skew_set():
    wl = syn.Workload("stress_small", T=300, H=256, I=64, E=48, k=8, Is=0, dense_I=64,
                      sigma_w=0.02, x_scale=8.0, stress=True, kind="prefill")
    inp = syn.make_site(wl, seed=0)
    cfg = S.SiteConfig(wl.H, wl.I, 0, wl.E, 0, wl.E, wl.k, wl.rsf, wl.limit)
    out = S.site_forward(inp, cfg, "prefill", tokens=inp["tie_tokens"])
    Sset = inp["skew_set"]
    for t in range(len(inp["tie_tokens"])):
        assert np.array_equal(out["ids"][t], Sset[:8])
        assert np.all(out["weights"][t] == 0.3125)      # 2.5 * 0.5 / (8 * 0.5)
    # every token's top-8 lies inside the skew set
    allout = S.site_forward(inp, cfg, "prefill")
    assert np.isin(allout["ids"], Sset).all()


def test_prefill_close_to_decode_w4a4_gap_is_small():
    wl, inp, cfg = _tiny()
    d = S.site_forward(inp, cfg, "decode")["y"]
    p = S.site_forward(inp, cfg, "prefill")["y"]
    rel = np.linalg.norm(p - d) / np.linalg.norm(d)
    assert 1e-4 < rel < 0.2


def test_permute_hand_worked_example():
    g = {ln[0]: [int(v) for v in ln[1:]] for ln in golden_lines("permute_example.txt")}
    ids = np.array(g["ids"]).reshape(3, 2)
    p = S.permute(ids, 4)
    for key in ("counts", "offsets", "sorted", "inv", "tile_offsets"):
        assert p[key].tolist() == g[key], key


def test_permute_invariants_random():
    rng = np.random.default_rng(2)
    ids = np.stack([rng.choice(40, 6, replace=False) for _ in range(500)])
    p = S.permute(ids, 40, rows_per_tile=128)
    flat = ids.reshape(-1)
    assert p["counts"].sum() == flat.size
    assert np.array_equal(np.sort(p["sorted"]), np.arange(flat.size))        # bijection
    assert np.array_equal(p["inv"][p["sorted"]], np.arange(flat.size))
    for e in range(40):
        seg = p["sorted"][p["offsets"][e]:p["offsets"][e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)           # stable


def test_combine_hand_example():
    r = np.array([[[1.0, 2.0], [0.5, -1.0], [0.25, 0.0]]])
    sh = np.array([[10.0, 20.0]])
    assert S.combine(r, sh).tolist() == [[11.75, 21.0]]
    assert S.combine(r).tolist() == [[1.75, 1.0]]


def test_dense_ffn_matches_torch_reference():
    rng = np.random.default_rng(0)
    xb = syn._to_bf16_bits(rng.standard_normal((3, 64)))
    wg, wu = syn.bf16_matrix(0, "dense_gate", 128, 64, 0.1), syn.bf16_matrix(0, "dense_up", 128, 64, 0.1)
    wd = syn.bf16_matrix(0, "dense_down", 64, 128, 0.1)
    tb = lambda a: torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).double()
    g, u = tb(xb) @ tb(wg).T, tb(xb) @ tb(wu).T
    ref = (torch.nn.functional.silu(torch.clamp(g, max=7.0)) * torch.clamp(u, -7.0, 7.0)) @ tb(wd).T
    assert np.allclose(S.dense_ffn(xb, wg, wu, wd, 7.0), ref.numpy(), rtol=1e-13, atol=1e-16)


# ------------------------------------------------------------------ readings 5, 6, 12

def test_zero_score_sum_gives_zero_weights():
    """Reading 5: no epsilon in the renormalisation; a zero denominator gives
    zero weights (never NaN). Logits of -1e30 give sigmoid scores of exactly 0."""
    l64 = np.full((3, 16), -1e30)
    ids = S.select_experts(l64.astype(np.float32), np.zeros(16, np.float32), 4)
    assert np.array_equal(ids, np.tile(np.arange(4, dtype=np.int32), (3, 1)))   # all keys equal: lowest indices
    w = S.routing_weights(l64, ids, 2.5)
    assert np.all(w == 0.0)


def test_nan_keys_rank_last_in_index_order():
    """Reading 6: a NaN key is chosen only when fewer finite keys than k are
    left, and NaN keys then go in index order."""
    E, k = 16, 4
    logits = np.zeros((2, E), np.float32)
    bias = np.zeros(E, np.float32)
    bias[[1, 5, 9]] = np.nan
    bias[[2, 3]] = 0.25
    ids = S.select_experts(logits, bias, k)
    assert ids[0].tolist() == [2, 3, 0, 4]            # finite keys first: 0.75 x2, then 0.5 by index
    nan_all = np.full(E, np.nan, np.float32)
    nan_all[7] = 0.0
    ids2 = S.select_experts(logits, nan_all, k)
    assert ids2[0].tolist() == [7, 0, 1, 2]          # the one finite key, then NaNs by index


def test_prefill_tokens_are_independent_of_their_batch():
    """Reading 12: the activation encoding's second-level scale is per token
    row, so a token's prefill output does not depend on the other tokens of
    the batch (chunked prefill equals whole prefill). A batch-wide scale would
    break this by far more than the fp64 tolerance."""
    wl, inp, cfg = _tiny()
    whole = S.site_forward(inp, cfg, "prefill")["y"]
    for t in range(wl.T):
        solo = S.site_forward(inp, cfg, "prefill", tokens=[t])["y"]
        assert np.allclose(solo[0], whole[t], rtol=1e-12, atol=1e-14)
    # and scaling one token's x (exactly, by a power of two) leaves the
    # others' outputs unchanged
    inp2 = dict(inp)
    x = np.asarray(inp["x"]).copy()
    x[0] = syn._to_bf16_bits(F.bf16_value(x[0]) * 4.0)
    inp2["x"] = x
    other = S.site_forward(inp2, cfg, "prefill")["y"]
    assert np.allclose(other[1:], whole[1:], rtol=1e-12, atol=1e-14)
