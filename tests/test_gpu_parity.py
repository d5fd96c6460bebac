"""GPU path vs the CPU oracle, element by element, through the C ABI.

Bar: expert indices, union lists, Q8_0 codes/scales and combine are bit-exact;
gate weights bit-exact; floating outputs within a max relative error of 2e-3
(|g - r| / max(|r|, rms of r's row)), with the bf16 output equal to the
round-to-nearest-even of the same call's fp32 output.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from synth.device import bits, device_layer, to_dev_bf16
from tests.helpers import layer_inputs, oracle_experts, rel_err_rows

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("quantized_mixture_experts_sigmoid_b200.moe")
TOL = 2e-3

SHAPES = {
    "tiny": synth.CONFIGS["tiny"],
    # several tiles and ragged tails: 17 hidden blocks, 9 h blocks, 37 tokens
    "ragged": synth.LayerShape("ragged", T=37, H=544, I=288, E=48, n_group=6, topk_group=3, top_k=5),
    # many tokens per expert: several staged token chunks per CTA plus a ragged one
    "crowded": synth.LayerShape("crowded", T=100, H=544, I=288, E=16, n_group=4, topk_group=2, top_k=5),
    "crowded_int8": synth.LayerShape("crowded_int8", T=100, H=544, I=288, E=16, n_group=4,
                                     topk_group=2, top_k=5, qtype=8),
    "crowded_int2": synth.LayerShape("crowded_int2", T=100, H=544, I=288, E=16, n_group=4,
                                     topk_group=2, top_k=5, qtype=2),
    # small batches take the fused persistent kernel (groups of a multiple of
    # 32 experts): ragged hidden sizes, T = 2, 3 and 4, 1 to 4 groups
    "fused_ragged": synth.LayerShape("fused_ragged", T=3, H=544, I=288, E=64, n_group=2, topk_group=1,
                                     top_k=5),
    "fused_ragged_int2": synth.LayerShape("fused_ragged_int2", T=2, H=576, I=160, E=128, n_group=4,
                                          topk_group=2, top_k=6, qtype=2),
    "fused_ragged_int8": synth.LayerShape("fused_ragged_int8", T=4, H=544, I=288, E=96, n_group=3,
                                          topk_group=2, top_k=5, qtype=8),
    # batches on the tensor cores: ragged N and K tails (I = 192, H = 320), partial 128-row
    # tiles of every height class, shared expert included; tc_multi gives every expert
    # about 160 pairs (two row tiles, the second partial) and the shared expert five
    "tc_small": synth.LayerShape("tc_small", T=40, H=256, I=128, E=16, n_group=4, topk_group=2, top_k=4),
    "tc_ragged": synth.LayerShape("tc_ragged", T=300, H=320, I=192, E=32, n_group=4, topk_group=2, top_k=6),
    "tc_multi": synth.LayerShape("tc_multi", T=640, H=320, I=192, E=16, n_group=4, topk_group=2, top_k=4),
    "decode": synth.CONFIGS["decode"],
    "verify": synth.CONFIGS["verify"],
    "verify_int8": synth.CONFIGS["verify_int8"],
    "decode_int2": synth.CONFIGS["decode"].with_(qtype=2, name="decode_int2"),
}
SMALL = ["tiny", "ragged", "crowded", "crowded_int8", "crowded_int2", "fused_ragged",
         "fused_ragged_int2", "fused_ragged_int8", "tc_small", "tc_ragged", "tc_multi"]
FULL = ["decode", "verify", "verify_int8", "decode_int2"]

_cache = {}


def layer(name):
    if name not in _cache:
        if len(_cache) >= 2:
            _cache.clear()
            torch.cuda.empty_cache()
        sh = SHAPES[name]
        _cache[name] = (sh, device_layer(sh))
    return _cache[name]


def gpu_route(sh, dev, x_bits):
    T = x_bits.shape[0]
    x = to_dev_bf16(x_bits)
    idx = torch.empty(T, sh.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, sh.top_k, dtype=torch.float32, device="cuda")
    ws = moe.workspace(moe.moe_route_workspace_bytes(T, dev["cfg"]))
    moe.moe_route(x, dev["W"], dev["bias"], dev["cfg"], idx, w, ws)
    return idx.cpu().numpy(), w.cpu().numpy()


def gpu_union(idx_np, E):
    T, K = idx_np.shape
    idx = torch.from_numpy(idx_np).cuda()
    nu = torch.zeros(1, dtype=torch.int32, device="cuda")
    uniq = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    offs = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    pt = torch.full((max(T * K, 1),), -1, dtype=torch.int32, device="cuda")
    ps = torch.full((max(T * K, 1),), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_union(idx, E, nu, uniq, offs, pt, ps, cnt, st)
    U = int(nu.item())
    return dict(n_unique=U, uniq=uniq[:U].cpu().numpy(), offsets=offs[:U + 1].cpu().numpy(),
                pair_tok=pt[:T * K].cpu().numpy(), pair_slot=ps[:T * K].cpu().numpy(),
                counts=cnt.cpu().numpy(), status=int(st.item()),
                dev=(nu, uniq, offs, pt, ps))


# ---------------------------------------------------------------- routing
@pytest.mark.parametrize("name", SMALL + ["decode", "verify"])
def test_route_bit_exact(name):
    sh, dev = layer(name)
    x, W, b = layer_inputs(sh)
    idx_g, w_g = gpu_route(sh, dev, x)
    idx_o, w_o, gap_e, gap_g = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    assert np.array_equal(idx_g, idx_o)
    assert np.array_equal(w_g.view(np.uint32), w_o.view(np.uint32))


def test_route_prefill_all_tokens_bit_exact():
    sh = synth.CONFIGS["prefill"]
    x, W, b = layer_inputs(sh)
    dev = dict(W=torch.from_numpy(W).cuda(), bias=torch.from_numpy(b).cuda(),
               cfg=moe.RouterCfg(sh.E, sh.n_group, sh.topk_group, sh.top_k, sh.rsf))
    idx_g, w_g = gpu_route(sh, dev, x)
    idx_o, w_o, gap_e, gap_g = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    assert np.array_equal(idx_g, idx_o)
    assert np.array_equal(w_g.view(np.uint32), w_o.view(np.uint32))
    un_g, un_o = gpu_union(idx_g, sh.E), O.union(idx_o, sh.E)
    for k in ("uniq", "offsets", "pair_tok", "pair_slot", "counts"):
        assert np.array_equal(un_g[k], un_o[k]), k


def test_route_degenerate_configs():
    # one group (no group limit), all groups kept, top_k = 1
    base = SHAPES["ragged"]
    for G, TG, K in [(1, 1, 4), (6, 6, 5), (6, 2, 1), (24, 3, 3)]:
        sh = base.with_(n_group=G, topk_group=TG, top_k=K)
        x, W, b = layer_inputs(sh)
        dev = dict(W=torch.from_numpy(W).cuda(), bias=torch.from_numpy(b).cuda(),
                   cfg=moe.RouterCfg(sh.E, G, TG, K, sh.rsf))
        idx_g, w_g = gpu_route(sh, dev, x)
        idx_o, w_o, _, _ = O.route(x, W, b, G, TG, K, sh.rsf)
        assert np.array_equal(idx_g, idx_o) and np.array_equal(w_g, w_o)


# ------------------------------------------------------------------ union
@pytest.mark.parametrize("T,E,K", [(1, 256, 8), (4, 16, 2), (37, 48, 5), (300, 256, 8), (513, 1024, 32),
                                   (2048, 256, 8)])
def test_union_bit_exact(T, E, K):
    rng = np.random.default_rng(T * 7 + E)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    g, o = gpu_union(idx, E), O.union(idx, E)
    assert g["n_unique"] == o["n_unique"] and g["status"] == 0
    for k in ("uniq", "offsets", "pair_tok", "pair_slot", "counts"):
        assert np.array_equal(g[k], o[k]), k


def test_union_all_tokens_same_experts_and_bad_index():
    idx = np.tile(np.array([[5, 1, 9]], np.int32), (70, 1))
    g, o = gpu_union(idx, 16), O.union(idx, 16)
    assert g["n_unique"] == 3
    for k in ("uniq", "offsets", "pair_tok", "pair_slot"):
        assert np.array_equal(g[k], o[k]), k
    bad = idx.copy()
    bad[3, 1] = 16  # outside [0, E): the kernel skips it and records the code
    g = gpu_union(bad, 16)
    assert g["status"] == moe.MOE_EDEVICE_INDEX


def test_union_leaves_out_a_repeated_expert():
    # a malformed row (one expert twice) is recorded and its repeat dropped; the pair lists
    # stay gap-free (equal to the lists of the same rows with the repeats emptied)
    rng = np.random.default_rng(5)
    T, E, K = 300, 64, 6
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    idx[7, 4] = idx[7, 1]
    idx[250, 5] = idx[250, 0]
    idx[299, 2] = idx[299, 3] = idx[299, 1]
    emptied = idx.copy()
    for t in range(T):
        for k in range(K):
            if idx[t, k] in idx[t, :k]:
                emptied[t, k] = -1
    assert (emptied == -1).sum() == 4
    g, o = gpu_union(idx, E), O.union(emptied, E)
    n = int(o["offsets"][o["n_unique"]])
    assert g["status"] == moe.MOE_EDEVICE_INDEX and n == T * K - 4
    assert g["n_unique"] == o["n_unique"]
    assert np.array_equal(g["uniq"], o["uniq"][:o["n_unique"]])
    assert np.array_equal(g["offsets"], o["offsets"][:o["n_unique"] + 1])
    assert np.array_equal(g["counts"], o["counts"])
    assert np.array_equal(g["pair_tok"][:n], o["pair_tok"][:n])
    assert np.array_equal(g["pair_slot"][:n], o["pair_slot"][:n])
    assert np.all(g["pair_tok"][n:] == 0) and np.all(g["pair_slot"][n:] == -1)


# ------------------------------------------------------------------- Q8_0
@pytest.mark.parametrize("n", [32, 544, 6144])
def test_q8_0_bit_exact(n):
    rng = np.random.default_rng(n)
    rows = 33
    v = (rng.standard_normal((rows, n)) * 10.0 ** rng.integers(-3, 3, (rows, 1))).astype(np.float32)
    v[1, :32] = 0.0
    v[2, :32] = 0.0
    v[2, 0] = 127.0
    v[2, 1:6] = [2.5, -2.5, 0.5, -0.5, 126.5]
    for dtype in ("f32", "bf16"):
        src = v if dtype == "f32" else synth.bf16_to_f32(synth.bf16_bits(v))
        t = torch.from_numpy(src).cuda() if dtype == "f32" else to_dev_bf16(synth.bf16_bits(v))
        q = torch.empty(rows, n, dtype=torch.int8, device="cuda")
        d = torch.empty(rows, n // 32, dtype=torch.float32, device="cuda")
        moe.moe_quantize_q8_0(t, q, d)
        qo, do = O.q8_0(src.reshape(-1))
        assert np.array_equal(q.cpu().numpy().reshape(-1), qo)
        assert np.array_equal(d.cpu().numpy().reshape(-1).view(np.uint32), do.view(np.uint32))


# ---------------------------------------------------------------- experts
def check_ffn(sh, dev, x, idx):
    un_o = O.union(idx, sh.E)
    un_g = gpu_union(idx, sh.E)
    T, K = idx.shape
    y = torch.zeros(T, K, sh.H, dtype=torch.float32, device="cuda")
    ws = moe.workspace(moe.moe_expert_ffn_workspace_bytes(dev["routed"], T, K))
    moe.moe_expert_ffn_q(dev["routed"], to_dev_bf16(x), K, un_g["dev"], y, ws)
    ex = oracle_experts(sh, un_o["uniq"])
    y_o = O.expert_ffn(ex, x, K, un_o)
    assert rel_err_rows(y.cpu().numpy(), y_o) <= TOL
    # shared expert in dense mode
    ys = torch.zeros(T, 1, sh.H, dtype=torch.float32, device="cuda")
    ws1 = moe.workspace(moe.moe_expert_ffn_workspace_bytes(dev["shared"], T, 1))
    moe.moe_expert_ffn_q(dev["shared"], to_dev_bf16(x), 1, None, ys, ws1)
    exs = oracle_experts(sh, [0], shared=True)
    ys_o = np.stack([O.expert_token(exs, 0, synth.bf16_to_f32(x[t])) for t in range(T)])
    assert rel_err_rows(ys.cpu().numpy()[:, 0], ys_o) <= TOL


@pytest.mark.parametrize("name", SMALL + FULL)
def test_expert_ffn_within_tolerance(name):
    sh, dev = layer(name)
    x, W, b = layer_inputs(sh)
    idx, _, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    check_ffn(sh, dev, x, idx)


# ---------------------------------------------------------------- combine
def test_combine_bit_exact():
    rng = np.random.default_rng(11)
    for T, K, H in [(1, 8, 6144), (37, 5, 544), (4, 1, 64)]:
        y = rng.standard_normal((T, K, H)).astype(np.float32)
        w = rng.uniform(0.05, 1.0, (T, K)).astype(np.float32)
        s = rng.standard_normal((T, H)).astype(np.float32)
        of, ob = O.combine(y, w, s)
        for shared in (True, False):
            of_n, ob_n = (of, ob) if shared else O.combine(y, w, None)
            out32 = torch.empty(T, H, dtype=torch.float32, device="cuda")
            out16 = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
            args = (torch.from_numpy(y).cuda(), torch.from_numpy(w).cuda(),
                    torch.from_numpy(s).cuda() if shared else None)
            moe.moe_combine(*args, out32)
            moe.moe_combine(*args, out16)
            assert np.array_equal(out32.cpu().numpy().view(np.uint32), of_n.view(np.uint32))
            assert np.array_equal(bits(out16), ob_n)


# ------------------------------------------------------------------ layer
def run_layer(sh, dev, x, shared=True):
    T = x.shape[0]
    xd = to_dev_bf16(x)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(T, dev["cfg"], dev["routed"], dev["shared"] if shared else None))
    out32 = torch.empty(T, sh.H, dtype=torch.float32, device="cuda")
    out16 = torch.empty(T, sh.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(T, sh.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, sh.top_k, dtype=torch.float32, device="cuda")
    sh_ex = dev["shared"] if shared else None
    moe.moe_layer_forward(xd, dev["W"], dev["bias"], dev["cfg"], dev["routed"], sh_ex, out32, ws, idx, w)
    moe.moe_layer_forward(xd, dev["W"], dev["bias"], dev["cfg"], dev["routed"], sh_ex, out16, ws)
    assert moe.moe_workspace_status(ws) == 0
    return out32.cpu().numpy(), bits(out16), idx.cpu().numpy(), w.cpu().numpy()


def check_layer(sh, dev, x, W, b, shared=True):
    of, ob, idx, w = run_layer(sh, dev, x, shared)
    idx_o, w_o, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    assert np.array_equal(idx, idx_o)
    assert np.array_equal(w.view(np.uint32), w_o.view(np.uint32))
    routed = oracle_experts(sh, np.unique(idx_o))
    shared_ex = oracle_experts(sh, [0], shared=True) if shared else None
    of_o, ob_o, _, _ = O.layer_forward(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, routed, shared_ex)
    err = rel_err_rows(of, of_o)
    assert err <= TOL, err
    assert np.array_equal(ob, synth.bf16_bits(of))  # bf16 output = RNE of the fp32 result
    assert rel_err_rows(synth.bf16_to_f32(ob), of_o) <= TOL + 2.0 ** -8
    return err


@pytest.mark.parametrize("name", SMALL + FULL)
def test_layer_forward_within_tolerance(name):
    sh, dev = layer(name)
    x, W, b = layer_inputs(sh)
    check_layer(sh, dev, x, W, b)


def test_layer_forward_without_shared_and_empty_batch():
    sh, dev = layer("ragged")
    x, W, b = layer_inputs(sh)
    check_layer(sh, dev, x, W, b, shared=False)
    ws = moe.workspace(1024)
    out = torch.empty(0, sh.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(to_dev_bf16(x[:0]), dev["W"], dev["bias"], dev["cfg"], dev["routed"],
                          dev["shared"], out, ws)


def test_tensor_core_path_without_shared_expert():
    # no shared rows: the gathered activation buffer and the tile list stop at the pairs
    sh, dev = layer("tc_multi")
    assert moe.moe_layer_path(sh.T, dev["cfg"], dev["routed"], None) == moe.PATH_TENSOR_CORE
    x, W, b = layer_inputs(sh)
    check_layer(sh, dev, x, W, b, shared=False)


def test_union_path_equals_per_token_path_on_gpu():
    # draft and verify must compute the same function (molayo1419.me, section
    # "정직하게 구현된 투기적 디코딩"): a token's output does not depend on which
    # other tokens share its batch-union pass
    sh, dev = layer("crowded")
    x, W, b = layer_inputs(sh)
    of_batch, _, _, _ = run_layer(sh, dev, x)
    for t in (0, 17, 99):
        of_one, _, _, _ = run_layer(sh, dev, x[t:t + 1])
        assert np.array_equal(of_one.view(np.uint32), of_batch[t:t + 1].view(np.uint32))


def test_union_path_equals_sub_batches_on_tensor_cores():
    # the same property on the tensor-core path: a token's output from a batch
    # of 300 equals its output from a batch of 5 (both above the fused size)
    sh, dev = layer("tc_ragged")
    x, W, b = layer_inputs(sh)
    of_batch, _, _, _ = run_layer(sh, dev, x)
    for t in (0, 17, 295):
        of_sub, _, _, _ = run_layer(sh, dev, x[t:t + 5])
        assert np.array_equal(of_sub.view(np.uint32), of_batch[t:t + 5].view(np.uint32))


FUSED = ["fused_ragged", "fused_ragged_int2", "fused_ragged_int8", "decode", "verify", "decode_int2"]
TENSOR_CORE = ["tc_small", "tc_ragged", "tc_multi"]


@pytest.mark.parametrize("name", FUSED + TENSOR_CORE + ["tiny", "ragged", "crowded_int8"])
def test_layer_forward_path(name):
    # small batches with groups of a multiple of 32 experts run as one fused
    # launch; int4 batches of more tokens on the tensor cores; other shapes take
    # the multi-kernel integer-dot path
    sh, dev = layer(name)
    path = moe.moe_layer_path(sh.T, dev["cfg"], dev["routed"], dev["shared"])
    x, W, b = layer_inputs(sh)
    xd = to_dev_bf16(x)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(sh.T, dev["cfg"], dev["routed"], dev["shared"]))
    out = torch.empty(sh.T, sh.H, dtype=torch.float32, device="cuda")
    n0 = moe.lib().moe_launch_count()
    moe.moe_layer_forward(xd, dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], out, ws)
    torch.cuda.synchronize()
    n = moe.lib().moe_launch_count() - n0
    assert moe.moe_workspace_status(ws) == 0
    if name in FUSED:
        assert path == moe.PATH_FUSED and n == 1
    elif name in TENSOR_CORE:
        assert path == moe.PATH_TENSOR_CORE and n > 1
    else:
        assert path == moe.PATH_GENERAL and n > 1


def test_layer_forward_repeated_calls_reuse_workspace():
    # the fused kernel's counters live in the workspace and reset themselves:
    # many calls in a row on one workspace give the same, correct result
    sh, dev = layer("decode")
    x, W, b = layer_inputs(sh)
    xd = to_dev_bf16(x)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(sh.T, dev["cfg"], dev["routed"], dev["shared"]))
    outs = []
    for i in range(20):
        out = torch.empty(sh.T, sh.H, dtype=torch.float32, device="cuda")
        moe.moe_layer_forward(xd, dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], out, ws)
        outs.append(out)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == 0  # also clears the counters
    # after a status clear the launch counter carries on: stale score slots of
    # earlier calls are never taken for this call's
    out = torch.empty(sh.T, sh.H, dtype=torch.float32, device="cuda")
    moe.moe_layer_forward(xd, dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], out, ws)
    outs.append(out)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == 0
    first = outs[0].cpu().numpy()
    for o in outs[1:]:
        assert np.array_equal(o.cpu().numpy().view(np.uint32), first.view(np.uint32))
    check_layer(sh, dev, x, W, b)


def test_route_nan_token_gets_no_expert():
    # a token whose scores are NaN cannot be routed: every slot gets index -1
    # and weight 0 (an empty slot, which moe_union leaves out), the workspace
    # router records the code, and the other tokens of the batch are routed as usual
    sh = SHAPES["ragged"]
    dev = dict(W=torch.from_numpy(synth.router_weight(sh)).cuda(),
               bias=torch.from_numpy(synth.router_bias(sh)).cuda(),
               cfg=moe.RouterCfg(sh.E, sh.n_group, sh.topk_group, sh.top_k, sh.rsf))
    x, W, b = layer_inputs(sh)
    x = x.copy()
    x[3, 7] = 0x7FC0  # bf16 quiet NaN
    idx_o, w_o, _, _ = O.route(np.delete(x, 3, axis=0), W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    for noalloc in (False, True):
        idx = torch.empty(sh.T, sh.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(sh.T, sh.top_k, dtype=torch.float32, device="cuda")
        xd = to_dev_bf16(x)
        if noalloc:
            moe.moe_route_noalloc(xd, dev["W"], dev["bias"], dev["cfg"], idx, w)
        else:
            ws = moe.workspace(moe.moe_route_workspace_bytes(sh.T, dev["cfg"]))
            moe.moe_route(xd, dev["W"], dev["bias"], dev["cfg"], idx, w, ws)
            assert moe.moe_workspace_status(ws) == moe.MOE_EDEVICE_INDEX
        ig, wg = idx.cpu().numpy(), w.cpu().numpy()
        assert np.all(ig[3] == -1) and np.all(wg[3] == 0.0)
        assert np.array_equal(np.delete(ig, 3, axis=0), idx_o)
        assert np.array_equal(np.delete(wg, 3, axis=0).view(np.uint32), w_o.view(np.uint32))
        g = gpu_union(ig, sh.E)
        assert g["status"] == 0 and 3 not in g["pair_tok"][:g["offsets"][-1]]
