"""GPU parity of the prefill path (W4A4 on tcgen05 block-scaled FP4) against
the CPU oracle, called through the C ABI: NVFP4 row encoding (bit-exact), the
re-tiled weight scales (bit-exact), the padded tile layout (bit-exact), the
grouped GEMM projections (against fp64 dot products of the GPU's own encoded
operands), and the whole prefill site on the tiny site and the H=4096, E=288
prefill / stress shapes."""
import numpy as np
import pytest
import torch

from helpers import assert_bf16_close, bf16_np, device_site, oracle_cfg, rel_l2, site_inputs, workload
from oracle import formats as OF
from oracle import site as OS

pytestmark = pytest.mark.gpu

capi = pytest.importorskip("routed_nvfp4_expert_b200.capi")


# ------------------------------------------------------------------ layout helpers (test side)

def sf_untile(atoms: np.ndarray, rows: int, K: int) -> np.ndarray:
    """512-byte scale atoms [ceil(rows/128)][K/64][512] -> row-major [rows, K/16]:
    the scale of row p, block b sits at ((p//128)*K/64 + b//4)*512 +
    (p%32)*16 + ((p%128)//32)*4 + b%4."""
    KB = K // 64
    p = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    off = ((p // 128) * KB + b // 4) * 512 + (p % 32) * 16 + ((p % 128) // 32) * 4 + b % 4
    return atoms.reshape(-1)[off]


TILE = 256   # rows of one padded-layout tile: every local expert starts on a multiple


def expected_tile_rows(ref_plan: dict, E: int, P: int, local) -> np.ndarray:
    lb, le = local
    out = np.full(P, -1, np.int32)
    tile = 0
    for e in range(E):
        c = int(ref_plan["counts"][e])
        if not (lb <= e < le) or c == 0:
            continue
        o = int(ref_plan["offsets"][e])
        out[tile * TILE: tile * TILE + c] = ref_plan["sorted"][o:o + c]
        tile += (c + TILE - 1) // TILE
    return out


def _arr(ptr, n, dtype=torch.int32):
    return capi.view_tensor(ptr, (n,), dtype).cpu().numpy().copy()


# ------------------------------------------------------------------ encoding

@pytest.mark.parametrize("rows,K", [(1, 256), (130, 1024), (300, 4096), (128, 64)])
def test_quantize_rows_bit_exact(rows, K):
    rng = np.random.default_rng(rows * 7 + K)
    x = rng.standard_normal((rows, K)).astype(np.float32) * rng.lognormal(0.0, 2.0, (rows, 1)).astype(np.float32)
    if rows > 3:
        x[1] = 0.0                                   # zero row: scale 0, every code and scale 0
        x[2, : K // 2] = 0.0                         # zero blocks inside a live row
        x[3] = -np.abs(x[3]) * 1e-3                  # small negatives: codes that round to -0
        x[3, 5] = -1000.0                            # one outlier sets the row scale
    bits = OF.f32_to_bf16_bits(x)
    src = capi.bf16_tensor(bits)
    tiles = (rows + 127) // 128
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.full((tiles * 128 * K // 16,), 0xAA, dtype=torch.uint8, device="cuda")
    scale = torch.empty((rows,), dtype=torch.float32, device="cuda")
    capi.nvfp4_quantize_rows(src, codes, sf, scale)
    rc, rs, rt = OF.quantize_rows_nvfp4(OF.bf16_value(bits).astype(np.float32))
    sfa = sf.cpu().numpy()
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(sf_untile(sfa, rows, K), rs)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), rt.view(np.uint32))
    if rows % 128:                                   # rows past the end of the last tile: zero scales
        pad = sf_untile(sfa, tiles * 128, K)[rows:]
        assert not pad.any()


def test_prepare_weights_bit_exact():
    wl = workload("tiny_t4")
    inp = site_inputs(wl)
    cfg = capi.config_for(wl)
    site = device_site(wl, inp)
    prep = capi.moe_prepare_weights(cfg, site).cpu().numpy()
    per = wl.E * wl.I * wl.H // 16
    r3 = (3 * per + 255) // 256 * 256
    assert prep.size == r3 + (wl.E * 3 * wl.H * 2 + 255) // 256 * 256
    # gate and up interleaved: atom rows 0..63 = gate rows 64 j.., 64..127 = up rows 64 j..
    got = sf_untile(prep[:2 * per], 2 * wl.E * wl.I, wl.H).reshape(wl.E, wl.I // 64, 2, 64, wl.H // 16)
    g = inp["gate_scales"].reshape(wl.E, wl.I // 64, 64, wl.H // 16)
    u = inp["up_scales"].reshape(wl.E, wl.I // 64, 64, wl.H // 16)
    assert np.array_equal(got[:, :, 0], g) and np.array_equal(got[:, :, 1], u)
    got = sf_untile(prep[2 * per:3 * per], wl.E * wl.H, wl.I)
    assert np.array_equal(got, inp["down_scales"].reshape(wl.E * wl.H, wl.I // 16))
    # router weight as three bf16 terms whose exact sum is the fp32 weight
    w3 = prep[r3:r3 + wl.E * 3 * wl.H * 2].view(np.uint16).reshape(wl.E, 3, wl.H)
    parts = OF.bf16_value(w3)
    assert np.array_equal(parts[:, 0] + parts[:, 1] + parts[:, 2], inp["router_w"].astype(np.float64))
    assert np.all(np.abs(parts[:, 1]) <= np.abs(parts[:, 2]) * 2.0 ** -7)     # order lo | mid | hi
    assert np.all(np.abs(parts[:, 0]) <= np.abs(parts[:, 1]) * 2.0 ** -7)


@pytest.mark.parametrize("T,E,k,local", [(4, 16, 4, (0, 16)), (1000, 16, 4, (0, 16)), (300, 32, 4, (8, 20)),
                                          (4096, 288, 8, (0, 288))])
def test_tile_rows_bit_exact(T, E, k, local):
    rng = np.random.default_rng(T * 3 + E)
    hot = rng.choice(E, min(E, 6), replace=False)
    ids = np.stack([rng.choice(hot if rng.random() < 0.5 and len(hot) >= k else E, k, replace=False)
                    for _ in range(T)]).astype(np.int32)
    cfg = capi.SiteConfig(256, 128, 0, E, local[0], local[1], k, 2.5, 7.0)
    buf = torch.empty(capi.moe_plan_size(cfg, T), dtype=torch.uint8, device="cuda")
    plan = capi.moe_plan_carve(cfg, T, buf)
    ws = capi.alloc_workspace(cfg, T, capi.PATH_DECODE)
    capi.moe_permute(cfg, torch.from_numpy(ids).cuda(), plan, ws)
    capi.moe_read_device_status(ws)
    P = capi.moe_padded_rows(cfg, T)
    assert P % TILE == 0
    got = _arr(plan.tile_rows, P)
    ref = expected_tile_rows(OS.permute(ids, E), E, P, local)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ site

def _prefill(wl, inp, local=None, x_bits=None):
    cfg = capi.config_for(wl, local)
    site = device_site(wl, inp)
    capi.moe_prepare_weights(cfg, site)
    xb = inp["x"] if x_bits is None else x_bits
    T = xb.shape[0]
    x = capi.bf16_tensor(xb)
    y = torch.empty_like(x)
    ws = capi.alloc_workspace(cfg, T, capi.PATH_PREFILL)
    capi.moe_forward(cfg, site, x, capi.PATH_PREFILL, y, ws)
    capi.moe_read_device_status(ws)
    v = capi.moe_workspace_views(cfg, T, capi.PATH_PREFILL, ws)
    return cfg, site, y, ws, v


def _site_state(wl, cfg, T, v):
    """Copy the prefill intermediates of the workspace to the host."""
    E, k, H, I = wl.E, wl.k, wl.H, wl.I
    P = capi.moe_padded_rows(cfg, T)
    ntiles = int(_arr(v.plan.tile_offsets, E + 1)[E])
    Pu = ntiles * TILE
    st = dict(P=P, Pu=Pu, tile_rows=_arr(v.plan.tile_rows, P), tile_offsets=_arr(v.plan.tile_offsets, E + 1),
              ids=_arr(v.ids, T * k).reshape(T, k), w=_arr(v.weights, T * k, torch.float32))
    st["xq"] = capi.view_tensor(v.xq_codes, (P, H // 2), torch.uint8).cpu().numpy()[:Pu]
    st["xsf"] = sf_untile(capi.view_tensor(v.xq_sf, (P * H // 16,), torch.uint8).cpu().numpy(), Pu, H)
    st["xts"] = capi.view_tensor(v.xq_scale, (P,), torch.float32).cpu().numpy()[:Pu]
    st["h"] = bf16_np(capi.view_tensor(v.h, (P, I), torch.bfloat16)[:Pu])
    st["hq"] = capi.view_tensor(v.hq_codes, (P, I // 2), torch.uint8).cpu().numpy()[:Pu]
    st["hsf"] = sf_untile(capi.view_tensor(v.hq_sf, (P * I // 16,), torch.uint8).cpu().numpy(), Pu, I)
    st["hts"] = capi.view_tensor(v.hq_scale, (P,), torch.float32).cpu().numpy()[:Pu]
    st["r_pad"] = bf16_np(capi.view_tensor(v.r, (P, H), torch.float32)[:Pu])
    return st


def _token_rows(cfg, wl, T, v):
    """The routed rows r[t, j] in token order, through moe_unpermute."""
    P = capi.moe_padded_rows(cfg, T)
    rows = capi.view_tensor(v.r, (P, wl.H), torch.float32)
    ids = capi.view_tensor(v.ids, (T, wl.k), torch.int32)
    out = torch.full((T, wl.k, wl.H), 3.0, dtype=torch.float32, device="cuda")
    capi.moe_unpermute(cfg, rows, T, v.plan, ids, out)
    return out


def _expert_of_rows(tile_offsets, Pu):
    mt = np.arange(Pu) // TILE
    return np.searchsorted(tile_offsets, mt, side="right") - 1


@pytest.mark.parametrize("T", [4, 33, 1000])
def test_prefill_encodings_and_gemms_tiny(T):
    """Each prefill step against the oracle on the GPU's own inputs: x codes
    bit-exact, h = clamped SwiGLU of the FP4 gate/up GEMM (fp64 dot products of
    the encoded operands), h codes bit-exact from the GPU's h, r = weight x the
    FP4 down GEMM."""
    wl = workload("tiny_t4", T)
    inp = site_inputs(wl)
    cfg, site, y, ws, v = _prefill(wl, inp)
    st = _site_state(wl, cfg, T, v)
    Pu, tr = st["Pu"], st["tile_rows"][:st["Pu"]]
    valid = tr >= 0
    # x encoded per assignment row (bit-exact), padding rows all zero
    xsrc = np.zeros((Pu, wl.H), np.float32)
    xsrc[valid] = OF.bf16_value(inp["x"][tr[valid] // wl.k]).astype(np.float32)
    rc, rs, rt = OF.quantize_rows_nvfp4(xsrc)
    assert np.array_equal(st["xq"], rc) and np.array_equal(st["xsf"], rs)
    assert np.array_equal(st["xts"].view(np.uint32), rt.view(np.uint32))
    # gate/up GEMM + clamped SwiGLU on the GPU's encoded x
    xdeq = OF.dequant_rows_nvfp4(st["xq"], st["xsf"], st["xts"])
    erow = _expert_of_rows(st["tile_offsets"], Pu)
    cache = OS.ExpertCache(inp)
    href = np.zeros((Pu, wl.I))
    for e in np.unique(erow):
        m = erow == e
        wg, wu, _ = cache.get(int(e))
        href[m] = OS.clamped_swiglu(xdeq[m] @ wg.T, xdeq[m] @ wu.T, wl.limit)
    d = np.abs(st["h"] - href)
    assert rel_l2(st["h"], href) < 4e-3
    assert np.all(d <= 2.0 ** -8 * np.abs(href) + 1e-4 * np.abs(href).max()), d.max()
    assert not st["h"][~valid].any()
    # h encoded per padded row from the GPU's own bf16 h (bit-exact)
    hsrc = np.where(valid[:, None], st["h"], 0.0).astype(np.float32)
    hc, hs, ht = OF.quantize_rows_nvfp4(hsrc)
    assert np.array_equal(st["hq"], hc) and np.array_equal(st["hsf"], hs)
    assert np.array_equal(st["hts"].view(np.uint32), ht.view(np.uint32))
    # down GEMM x routing weight, rows in the padded tile order (padding rows zero)
    hdeq = OF.dequant_rows_nvfp4(st["hq"], st["hsf"], st["hts"])
    rref = np.zeros((Pu, wl.H))
    for e in np.unique(erow):
        m = (erow == e) & valid
        _, _, wd = cache.get(int(e))
        rref[m] = st["w"][tr[m], None] * (hdeq[m] @ wd.T)
    r = st["r_pad"]
    d = np.abs(r - rref)
    assert rel_l2(r, rref) < 4e-3
    assert np.all(d <= 2.0 ** -8 * np.abs(rref) + 1e-4 * np.abs(rref).max()), d.max()
    assert not r[~valid].any()
    # unpermute: token order, remote/padding never read
    rt = bf16_np(_token_rows(cfg, wl, T, v)).reshape(T * wl.k, wl.H)
    assert np.array_equal(rt[tr[valid]], r[valid])


def test_grouped_gemm_entry_point_matches_forward():
    wl = workload("tiny_t4", 300)
    inp = site_inputs(wl)
    cfg, site, y, ws, v = _prefill(wl, inp)
    T, P = wl.T, capi.moe_padded_rows(cfg, wl.T)
    xq = capi.view_tensor(v.xq_codes, (P, wl.H // 2), torch.uint8)
    xsf = capi.view_tensor(v.xq_sf, (P * wl.H // 16,), torch.uint8)
    xts = capi.view_tensor(v.xq_scale, (P,), torch.float32)
    hq = capi.view_tensor(v.hq_codes, (P, wl.I // 2), torch.uint8)
    hsf = capi.view_tensor(v.hq_sf, (P * wl.I // 16,), torch.uint8)
    hts = capi.view_tensor(v.hq_scale, (P,), torch.float32)
    wts = capi.view_tensor(v.weights, (T * wl.k,), torch.float32)
    ws2 = capi.alloc_workspace(cfg, T, capi.PATH_PREFILL)
    h2 = torch.zeros((P, wl.I), dtype=torch.bfloat16, device="cuda")
    capi.nvfp4_grouped_gemm(cfg, capi.PROJ_GATE_UP, xq, xsf, xts, T, v.plan, wts, site, h2, ws2)
    r2 = torch.full((P, wl.H), 7.0, dtype=torch.float32, device="cuda")
    capi.nvfp4_grouped_gemm(cfg, capi.PROJ_DOWN, hq, hsf, hts, T, v.plan, wts, site, r2, ws2)
    capi.moe_read_device_status(ws2)
    ntiles = int(_arr(v.plan.tile_offsets, wl.E + 1)[wl.E])
    h = capi.view_tensor(v.h, (P, wl.I), torch.bfloat16)
    r = capi.view_tensor(v.r, (P, wl.H), torch.float32)
    assert torch.equal(h2[:ntiles * TILE], h[:ntiles * TILE])
    assert torch.equal(r2[:ntiles * TILE], r[:ntiles * TILE])
    # the fused unpermute + combine equals unpermute then moe_combine, and y
    ids = capi.view_tensor(v.ids, (T, wl.k), torch.int32)
    sh = capi.view_tensor(v.shared, (T, wl.H), torch.float32)
    y2 = torch.empty_like(y)
    capi.moe_unpermute_combine(cfg, r, T, v.plan, ids, sh, y2)
    assert torch.equal(y2, y)
    rt = _token_rows(cfg, wl, T, v)
    y3 = torch.empty_like(y)
    capi.moe_combine(rt, sh, y3)
    assert torch.equal(y3, y)


@pytest.mark.parametrize("name,T", [("tiny_t4", None), ("tiny_t4", 33), ("tiny_t4", 1000), ("prefill_t4096", None),
                                    ("stress_t16384", None)])
def test_moe_forward_prefill_matches_oracle(name, T):
    wl = workload(name, T)
    inp = site_inputs(wl)
    cfg, site, y, ws, v = _prefill(wl, inp)
    lg = capi.view_tensor(v.logits, (wl.T, wl.E), torch.float32).cpu().numpy()
    if wl.T <= 40:
        tokens = np.arange(wl.T)
    else:
        tokens = np.random.default_rng(2).choice(wl.T, 12, replace=False)
        if wl.stress:                                 # include exactly tied tokens
            tokens = np.unique(np.concatenate([tokens, inp["tie_tokens"][:4]]))
    ref = OS.site_forward(inp, oracle_cfg(wl), "prefill", tokens=tokens, gpu_logits=lg[tokens], want_parts=True)
    if wl.stress:                                     # x8 activations: the clamp fires on the tails
        assert ref["clamp_fired"] > 0.01 * ref["clamp_total"]
    # logits (tensor-core split-bf16 GEMM at T >= 128): 1e-5 of the token's largest logit
    rl = ref["logits"]
    scale = np.maximum(np.abs(rl), np.abs(rl).max(axis=1, keepdims=True))
    assert np.all(np.abs(lg[tokens] - rl) <= 1e-5 * scale), np.abs(lg[tokens] - rl).max()
    ids = capi.view_tensor(v.ids, (wl.T, wl.k), torch.int32).cpu().numpy()
    assert np.array_equal(ids[tokens], ref["ids"])
    got = bf16_np(y)[tokens]
    if not wl.stress:
        assert_bf16_close(got, ref["y"], what=f"{wl.name} y")
        r = _token_rows(cfg, wl, wl.T, v)
        assert_bf16_close(bf16_np(r)[tokens], ref["r"], what="r")
        return
    # x8 activations put many h values next to an NVFP4 code boundary. The h
    # encoding is a decision on the GPU's bf16 h, whose GEMM sum rounds in
    # another order than the oracle's fp64 h, so the two sides may pick
    # neighbouring codes there. The GPU's h is held to the GEMM tolerance
    # against the oracle; y to the elementwise gate against the oracle's down
    # projection and combine of the GPU's own h encoding, and to the relative
    # L2 bound against the independent oracle.
    prow, pids = _assignment_rows(cfg, wl, v, tokens)
    live = prow >= 0
    P = capi.moe_padded_rows(cfg, wl.T)
    sel = np.where(live, prow, 0).reshape(-1)
    hg = bf16_np(capi.view_tensor(v.h, (P, wl.I), torch.bfloat16)[torch.from_numpy(sel).cuda().long()])
    cache = OS.ExpertCache(inp)
    xdeq = OS.prefill_activation(inp["x"][tokens])
    for ti, j in zip(*np.nonzero(live)):
        wg, wu, _ = cache.get(int(pids[ti, j]))
        href = OS.clamped_swiglu(wg @ xdeq[ti], wu @ xdeq[ti], wl.limit)
        hrow = hg[ti * wl.k + j]
        d = np.abs(hrow - href)
        assert np.all(d <= 2.0 ** -8 * np.abs(href) + 1e-4 * np.abs(href).max()), (ti, j, d.max())
    yh = _y_from_gpu_h(wl, cfg, v, inp, tokens, prow, pids, ref)
    assert_bf16_close(got, yh, what=f"{wl.name} y (oracle down on the GPU's h codes)")
    assert rel_l2(got, ref["y"]) < 5e-3


def _assignment_rows(cfg, wl, v, tokens):
    """Padded-layout row of each assignment (t, j) of the given tokens (-1 for
    a remote expert), and the ids: expert e's segment starts at tile
    tile_offsets[e], in the stable sorted order of the plan."""
    E, k, T = wl.E, wl.k, wl.T
    ids = _arr(v.ids, T * k).reshape(T, k)[tokens]
    inv = _arr(v.plan.inv, T * k).reshape(T, k)[tokens]
    offs = _arr(v.plan.offsets, E + 1)
    toffs = _arr(v.plan.tile_offsets, E + 1)
    local = (ids >= cfg.local_begin) & (ids < cfg.local_end)
    rows = toffs[ids] * TILE + (inv - offs[ids])
    return np.where(local, rows, -1), ids


def _y_from_gpu_h(wl, cfg, v, inp, tokens, prow, ids, ref):
    """The oracle's down projection, routing weights and combine applied to the
    GPU's NVFP4 encoding of h for the given tokens."""
    P = capi.moe_padded_rows(cfg, wl.T)
    sel = np.where(prow >= 0, prow, 0).reshape(-1)
    codes = capi.view_tensor(v.hq_codes, (P, wl.I // 2), torch.uint8)[torch.from_numpy(sel).cuda().long()]
    atoms = capi.view_tensor(v.hq_sf, (P * wl.I // 16,), torch.uint8).cpu().numpy()
    KB = wl.I // 64
    pp, b = sel[:, None], np.arange(wl.I // 16)[None, :]
    sf = atoms[((pp // 128) * KB + b // 4) * 512 + (pp % 32) * 16 + ((pp % 128) // 32) * 4 + b % 4]
    ts = capi.view_tensor(v.hq_scale, (P,), torch.float32).cpu().numpy()[sel]
    hdeq = OF.dequant_rows_nvfp4(codes.cpu().numpy(), sf, ts).reshape(len(tokens), wl.k, wl.I)
    cache = OS.ExpertCache(inp)
    r = np.zeros((len(tokens), wl.k, wl.H))
    for ti, j in zip(*np.nonzero(prow >= 0)):
        _, _, wd = cache.get(int(ids[ti, j]))
        r[ti, j] = ref["weights"][ti, j] * (wd @ hdeq[ti, j])
    return OS.combine(r, ref["shared"])


def test_prefill_is_deterministic_and_chunk_invariant():
    """Per-row encodings keep every token independent of its batch: the routed
    rows r of a chunked prefill equal those of the whole batch bit for bit."""
    wl = workload("tiny_t4", 600)
    inp = site_inputs(wl)
    cfg1, _, y1, _, v1 = _prefill(wl, inp)
    r1 = _token_rows(cfg1, wl, wl.T, v1)
    _, _, y2, _, _ = _prefill(wl, inp)
    assert torch.equal(y1, y2)
    cut = 217
    cfga, _, ya, _, va = _prefill(wl, inp, x_bits=inp["x"][:cut])
    ra = _token_rows(cfga, wl, cut, va)
    cfgb, _, yb, _, vb = _prefill(wl, inp, x_bits=inp["x"][cut:])
    rb = _token_rows(cfgb, wl, wl.T - cut, vb)
    assert torch.equal(torch.cat([ra, rb]), r1)
    assert_bf16_close(bf16_np(torch.cat([ya, yb])), bf16_np(y1), what="chunked y")


@pytest.mark.parametrize("T", [4, 300])
def test_prefill_local_range_masks_remote_experts(T):
    wl = workload("tiny_t4", T)
    inp = site_inputs(wl)
    local = (5, 11)
    cfg, site, y, ws, v = _prefill(wl, inp, local=local)
    lg = capi.view_tensor(v.logits, (wl.T, wl.E), torch.float32).cpu().numpy()
    tokens = np.arange(min(T, 40))
    ref = OS.site_forward(inp, oracle_cfg(wl, local), "prefill", tokens=tokens, gpu_logits=lg[tokens],
                          want_parts=True)
    assert_bf16_close(bf16_np(y)[tokens], ref["y"], what="local y")
    ids = capi.view_tensor(v.ids, (wl.T, wl.k), torch.int32).cpu().numpy()
    r = bf16_np(_token_rows(cfg, wl, wl.T, v))
    remote = (ids < local[0]) | (ids >= local[1])
    assert remote.any() and not r[remote].any()


@pytest.mark.parametrize("name,T", [("tiny_t4", 33), ("mid", 300)])
def test_prefill_on_quantised_bank(name, T):
    """The prefill on expert banks made by quantising Gaussian weights (block
    scales up to 448) matches the oracle."""
    from helpers import with_quantised_banks
    from routed_nvfp4_expert_b200 import synthetic as syn
    if name == "mid":
        wl = syn.Workload("mid", T=T, H=1024, I=512, E=32, k=8, Is=512, dense_I=64, sigma_w=0.0064, kind="prefill")
    else:
        wl = workload(name, T)
    inp = with_quantised_banks(wl, site_inputs(wl))
    cfg = capi.config_for(wl)
    site = capi.site_to_device(inp)
    capi.moe_prepare_weights(cfg, site)
    x = capi.bf16_tensor(inp["x"])
    y = torch.empty_like(x)
    ws = capi.alloc_workspace(cfg, wl.T, capi.PATH_PREFILL)
    capi.moe_forward(cfg, site, x, capi.PATH_PREFILL, y, ws)
    capi.moe_read_device_status(ws)
    v = capi.moe_workspace_views(cfg, wl.T, capi.PATH_PREFILL, ws)
    lg = capi.view_tensor(v.logits, (wl.T, wl.E), torch.float32).cpu().numpy()
    tokens = np.arange(min(wl.T, 24))
    ref = OS.site_forward(inp, oracle_cfg(wl), "prefill", tokens=tokens, gpu_logits=lg[tokens])
    assert_bf16_close(bf16_np(y)[tokens], ref["y"], what=f"{name} quantised-bank prefill y")


# ------------------------------------------------------------------ W4A16 prefill (the pages' numerics)

def _prefill_w4(wl, inp, local=None):
    cfg = capi.config_for(wl, local)
    site = device_site(wl, inp)
    capi.moe_prepare_weights(cfg, site)
    x = capi.bf16_tensor(inp["x"])
    y = torch.empty_like(x)
    ws = capi.alloc_workspace(cfg, wl.T, capi.PATH_PREFILL_W4A16)
    capi.moe_forward(cfg, site, x, capi.PATH_PREFILL_W4A16, y, ws)
    capi.moe_read_device_status(ws)
    v = capi.moe_workspace_views(cfg, wl.T, capi.PATH_PREFILL_W4A16, ws)
    return cfg, site, y, ws, v


@pytest.mark.parametrize("name,T", [("tiny_t4", None), ("tiny_t4", 33), ("tiny_t4", 1000), ("prefill_t4096", None),
                                    ("stress_t16384", None)])
def test_w4a16_prefill_matches_oracle(name, T):
    """The W4A16 prefill computes the decode numerics (bf16 x straight into
    the NVFP4 experts, no activation quantisation) as a grouped GEMM: it holds
    the output gate against the oracle's W4A16 site."""
    wl = workload(name, T)
    inp = site_inputs(wl)
    cfg, site, y, ws, v = _prefill_w4(wl, inp)
    lg = capi.view_tensor(v.logits, (wl.T, wl.E), torch.float32).cpu().numpy()
    if wl.T <= 40:
        tokens = np.arange(wl.T)
    else:
        tokens = np.random.default_rng(3).choice(wl.T, 12, replace=False)
        if wl.stress:
            tokens = np.unique(np.concatenate([tokens, inp["tie_tokens"][:4]]))
    ref = OS.site_forward(inp, oracle_cfg(wl), "decode", tokens=tokens, gpu_logits=lg[tokens], want_parts=True)
    ids = capi.view_tensor(v.ids, (wl.T, wl.k), torch.int32).cpu().numpy()
    assert np.array_equal(ids[tokens], ref["ids"])
    got = bf16_np(y)[tokens]
    assert_bf16_close(got, ref["y"], what=f"{wl.name} W4A16 y")
    assert rel_l2(got, ref["y"]) < 5e-3
    r = _token_rows(cfg, wl, wl.T, v)
    assert_bf16_close(bf16_np(r)[tokens], ref["r"], what="W4A16 r")


def test_w4a16_entry_point_matches_forward():
    wl = workload("tiny_t4", 300)
    inp = site_inputs(wl)
    cfg, site, y, ws, v = _prefill_w4(wl, inp)
    T, P = wl.T, capi.moe_padded_rows(cfg, wl.T)
    xa = capi.view_tensor(v.xq_codes, (P, wl.H), torch.float16)
    xs = capi.view_tensor(v.xq_scale, (P,), torch.float32)
    h = capi.view_tensor(v.h, (P, wl.I), torch.float16)
    r = capi.view_tensor(v.r, (P, wl.H), torch.float32)
    wts = capi.view_tensor(v.weights, (T * wl.k,), torch.float32)
    ws2 = capi.alloc_workspace(cfg, T, capi.PATH_PREFILL_W4A16)
    h2 = torch.zeros((P, wl.I), dtype=torch.float16, device="cuda")
    capi.nvfp4_grouped_gemm_w4a16(cfg, capi.PROJ_GATE_UP, xa, xs, T, v.plan, wts, site, h2, ws2)
    r2 = torch.full((P, wl.H), 7.0, dtype=torch.float32, device="cuda")
    capi.nvfp4_grouped_gemm_w4a16(cfg, capi.PROJ_DOWN, h, None, T, v.plan, wts, site, r2, ws2)
    capi.moe_read_device_status(ws2)
    used = int(_arr(v.plan.tile_offsets, wl.E + 1)[wl.E]) * TILE
    assert torch.equal(h2[:used], h[:used])
    assert torch.equal(r2[:used], r[:used])
    # the gathered x rows: f16 of x times a power of two, exactly; padding rows zero
    tr = _arr(v.plan.tile_rows, P)[:used]
    xs_np = xs.cpu().numpy()[:used]
    xa_np = xa.float().cpu().numpy().astype(np.float64)[:used]
    valid = tr >= 0
    want = OF.bf16_value(inp["x"][tr[valid] // wl.k])
    assert np.array_equal(xa_np[valid] * xs_np[valid, None].astype(np.float64), want)
    assert not xa_np[~valid].any()


def test_w4a16_prefill_local_range_masks_remote_experts():
    wl = workload("tiny_t4", 300)
    inp = site_inputs(wl)
    local = (5, 11)
    cfg, site, y, ws, v = _prefill_w4(wl, inp, local=local)
    lg = capi.view_tensor(v.logits, (wl.T, wl.E), torch.float32).cpu().numpy()
    tokens = np.arange(40)
    ref = OS.site_forward(inp, oracle_cfg(wl, local), "decode", tokens=tokens, gpu_logits=lg[tokens])
    assert_bf16_close(bf16_np(y)[tokens], ref["y"], what="W4A16 local y")
