"""Expert parallelism on one GPU: G ranks emulated as G handles in one process,
whose kernels address each other's workspaces, run in lockstep on one stream
(the stream order stands in for the barriers between the steps).

Each rank holds mN / G routed experts and routes its own tokens.  Its output
must equal, bit for bit, the single-GPU layer's output on the same tokens:
every row is computed by the same kernels in the same order (the routing of a
token, a routed row's GEMMs, the k-ordered sum), only the place of the rows
differs.  A sample of tokens is also compared with the oracle directly.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fine_grained_shared_b200 import moe as B
from tests import harness as H

pytestmark = pytest.mark.gpu

LS = W.LayerShape

# (shape over all ranks' tokens, G, tokens per rank, node limit, flags)
CASES = {
    "g2_softmax": (LS("ep_g2", T=633, d=256, N=16, I=128, K=4, Ks=1, Is=128, sigma=0.05, seed=81), 2,
                   [300, 333], None, 0),
    # one rank without tokens, one on the CUDA-core router (T <= 256); a token reaches at most 2 ranks
    "g4_sigmoid_node_limited": (LS("ep_g4", T=515, d=384, N=32, I=256, K=4, Ks=0, Is=0, gate="sigmoid",
                                   sigma=0.03, bias="uniform", seed=82), 4, [257, 129, 0, 129], (4, 2), 0),
    "g8_k8_no_residual": (LS("ep_g8", T=1100, d=256, N=64, I=128, K=8, Ks=2, Is=128, sigma=0.05,
                             bias="normal", seed=83), 8, [100, 200, 65, 135, 300, 100, 100, 100], None,
                          B.MOE_FLAG_NO_RESIDUAL),
}


def _split(shape, Ts):
    assert sum(Ts) == shape.T
    return np.cumsum([0] + Ts)


def _layers(shape, dev, G, node_limit, flags, max_tokens):
    per = shape.N // G
    shared = (dev["ws_gate"], dev["ws_up"], dev["ws_down"]) if shape.Ks else None
    layers = []
    for r in range(G):
        layer = B.ExpertParallelLayer(ep_ranks=G, ep_rank=r, d_model=shape.d, n_routed=shape.N, d_ff=shape.I,
                                      n_shared=shape.Ks, d_ff_shared=shape.Is, max_tokens=max_tokens,
                                      max_k=shape.K, gate=shape.gate, flags=flags, node_limit=node_limit)
        sl = slice(r * per, (r + 1) * per)
        layer.set_weights(dev["router"], (dev["w_gate"][sl], dev["w_up"][sl], dev["w_down"][sl]), shared,
                          logit_bias=dev["logit_bias"], select_bias=dev["select_bias"])
        layers.append(layer)
    B.connect_emulated(layers)
    return layers


def _single(shape, dev, node_limit, flags, max_tokens):
    layer = B.MoELayer(d_model=shape.d, n_routed=shape.N, d_ff=shape.I, n_shared=shape.Ks, d_ff_shared=shape.Is,
                       max_tokens=max_tokens, max_k=shape.K, gate=shape.gate, flags=flags, node_limit=node_limit)
    shared = (dev["ws_gate"], dev["ws_up"], dev["ws_down"]) if shape.Ks else None
    layer.set_weights(dev["router"], (dev["w_gate"], dev["w_up"], dev["w_down"]), shared,
                      logit_bias=dev["logit_bias"], select_bias=dev["select_bias"])
    return layer


def _run_case(shape, G, Ts, node_limit, flags, oracle_rows_per_rank=6, repeats=2):
    host, dev = H.device_inputs(shape)
    cut = _split(shape, Ts)
    xs = [dev["x"][cut[r]:cut[r + 1]] for r in range(G)]
    layers = _layers(shape, dev, G, node_limit, flags, max(Ts))
    single = _single(shape, dev, node_limit, flags, max(Ts))
    for _ in range(repeats):                       # a second forward reuses every buffer and counter
        outs = B.forward_emulated(layers, xs, shape.K)
        for r, layer in enumerate(layers):
            assert layer.status() == B.MOE_OK, B.status_string(layer.status())
    for r in range(G):
        if Ts[r] == 0:
            continue
        want = H.run(single, xs[r], shape.K)
        assert torch.equal(outs[r].view(torch.int16), want.view(torch.int16)), f"rank {r}: differs from 1 GPU"
        # the rank's routing is the single-GPU routing of its tokens
        idx, gate = (t.cpu() for t in layers[r].routing(Ts[r], shape.K)[:2])
        idx1, gate1 = (t.cpu() for t in single.routing(Ts[r], shape.K)[:2])
        assert torch.equal(idx, idx1) and torch.equal(gate, gate1)
        per = shape.N // G
        if node_limit is not None:
            assert all(len({e // per for e in row}) <= node_limit[1] for row in idx.tolist())
    # a few tokens of every rank against the oracle
    rows = np.concatenate([cut[r] + np.arange(min(oracle_rows_per_rank, Ts[r])) for r in range(G)])
    ref = O.route(host["x"][rows], host["router"], shape.K, shape.gate, host["logit_bias"], host["select_bias"],
                  node_limit=node_limit)
    h, _ = O.moe_forward(host["x"][rows], host["router"], shape.K, H.oracle_experts(shape, host),
                         H.oracle_shared(shape, host), gate_kind=shape.gate, logit_bias=host["logit_bias"],
                         select_bias=host["select_bias"], routing=ref, flags=flags)
    got = torch.cat(outs).float().cpu().numpy()[rows].astype(np.float64)
    H.compare_output(got, h, f"{shape.name} expert-parallel output", term=flags != 0)
    for layer in layers:
        layer.close()
    single.close()


@pytest.mark.parametrize("case", sorted(CASES))
def test_expert_parallel_layer_equals_the_single_gpu_layer(case):
    shape, G, Ts, node_limit, flags = CASES[case]
    _run_case(shape, G, Ts, node_limit, flags)


def test_expert_parallel_16b_prefill_on_four_ranks():
    """The 16B layer's prefill batch, 4096 tokens on each of 4 ranks of 16 experts."""
    shape = W.CONFIGS["16b_prefill"]
    _run_case(shape, 4, [4096] * 4, None, 0, repeats=1)


def test_expert_parallel_v3_on_eight_ranks_node_limited():
    """The V3 layer, 512 tokens on each of 8 ranks of 32 experts, each token's experts on at most
    4 ranks (the report's node-limited routing with a rank per node)."""
    shape = W.CONFIGS["v3"]
    _run_case(shape, 8, [512] * 8, (8, 4), 0, repeats=1, oracle_rows_per_rank=2)


@pytest.mark.parametrize("G,Ts", [(2, [300, 333]), (4, [257, 0, 129, 200])])
def test_expert_parallel_fp8_layer_equals_the_single_gpu_fp8_layer(G, Ts):
    """The FP8 layer split over G ranks: the dispatch sends each row's E4M3 codes and scale bytes
    (quantized once, 1 x 128 groups, as moe_forward_fp8 does), the owners run the FP8 expert GEMMs;
    every rank's output bit-identical to moe_forward_fp8 on its tokens."""
    shape = LS("ep_fp8", T=sum(Ts), d=256, N=16, I=256, K=4, Ks=1, Is=128, sigma=0.05, seed=86)
    host, dev = H.device_inputs(shape)
    cut = _split(shape, Ts)
    xs = [dev["x"][cut[r]:cut[r + 1]] for r in range(G)]
    qw = tuple(B.quantize_fp8_blocks(dev[k]) for k in ("w_gate", "w_up", "w_down"))
    qs = tuple(B.quantize_fp8_blocks(dev[k]) for k in ("ws_gate", "ws_up", "ws_down"))
    per = shape.N // G
    layers = []
    for r in range(G):
        layer = B.ExpertParallelLayer(ep_ranks=G, ep_rank=r, d_model=shape.d, n_routed=shape.N, d_ff=shape.I,
                                      n_shared=shape.Ks, d_ff_shared=shape.Is, max_tokens=max(Ts), max_k=shape.K,
                                      flags=B.MOE_FLAG_FP8)
        layer.set_weights(dev["router"], (dev["w_gate"], dev["w_up"], dev["w_down"]),
                          (dev["ws_gate"], dev["ws_up"], dev["ws_down"]))
        sl = slice(r * per, (r + 1) * per)
        layer.set_weights_fp8(tuple((c[sl], sc[sl]) for c, sc in qw), qs)
        layers.append(layer)
    B.connect_emulated(layers)
    outs = B.forward_emulated(layers, xs, shape.K)
    single = B.MoELayer(d_model=shape.d, n_routed=shape.N, d_ff=shape.I, n_shared=shape.Ks, d_ff_shared=shape.Is,
                        max_tokens=max(Ts), max_k=shape.K, flags=B.MOE_FLAG_FP8)
    single.set_weights(dev["router"], (dev["w_gate"], dev["w_up"], dev["w_down"]),
                       (dev["ws_gate"], dev["ws_up"], dev["ws_down"]))
    single.set_weights_fp8(qw, qs)
    for r in range(G):
        assert layers[r].status() == B.MOE_OK
        if Ts[r] == 0:
            continue
        want = single.forward_fp8(xs[r], shape.K)
        assert single.status() == B.MOE_OK
        assert torch.equal(outs[r].view(torch.int16), want.view(torch.int16)), f"rank {r}"
    # on an FP8 handle the bf16 experts step is refused (the rows arrived as FP8 codes)
    layers[0].route(xs[0], shape.K)
    layers[0].dispatch()
    assert B.moe_ep_experts(layers[0].h, layers[0].experts, layers[0].shared, None) == B.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    for layer in layers:
        layer.close()
    single.close()


def test_expert_parallel_calls_check_their_order_and_peers():
    shape = LS("ep_args", T=256, d=128, N=8, I=64, K=2, Ks=1, Is=64, sigma=0.05, seed=84)
    host, dev = H.device_inputs(shape)
    layers = _layers(shape, dev, 2, None, 0, 128)
    x = dev["x"][:128]
    with pytest.raises(B.MoEError) as e:
        layers[0].dispatch()
    assert e.value.status == B.MOE_ERR_INVALID_ARG               # dispatch before route
    st, _ = B.MoELayer.forward(layers[0], x, 2, check=False)
    assert st == B.MOE_ERR_UNSUPPORTED                           # the single-GPU forward
    layers[0].route(x, 2)
    with pytest.raises(B.MoEError):
        layers[0].experts_step()                                 # experts before dispatch
    ws = [layer.workspace() for layer in layers]
    with pytest.raises(B.MoEError):
        layers[0].set_peers([ws[1], ws[1]])                      # its own entry is not its workspace
    fresh = B.ExpertParallelLayer(ep_ranks=2, ep_rank=1, d_model=shape.d, n_routed=shape.N, d_ff=shape.I,
                                  n_shared=shape.Ks, d_ff_shared=shape.Is, max_tokens=128, max_k=shape.K)
    fresh.set_weights(dev["router"], (dev["w_gate"][4:], dev["w_up"][4:], dev["w_down"][4:]),
                      (dev["ws_gate"], dev["ws_up"], dev["ws_down"]))
    fresh.route(x, 2)
    with pytest.raises(B.MoEError):
        fresh.dispatch()                                         # no peers yet
    fresh.close()
    # a normal forward after all of that
    outs = B.forward_emulated(layers, [x, dev["x"][128:]], 2)
    single = _single(shape, dev, None, 0, 128)
    for r, xr in enumerate((x, dev["x"][128:])):
        assert torch.equal(outs[r].view(torch.int16), H.run(single, xr, 2).view(torch.int16))


def test_expert_parallel_rank_timeout_is_reported_on_that_rank():
    """A bounded wait that runs out in one rank's grouped GEMM (the test-only flag on rank 0):
    rank 0 reports MOE_ERR_TIMEOUT, the other rank finishes, and both run normally afterwards."""
    shape = LS("ep_timeout", T=600, d=256, N=16, I=128, K=4, Ks=1, Is=128, sigma=0.05, seed=85)
    host, dev = H.device_inputs(shape)
    xs = [dev["x"][:300], dev["x"][300:]]
    per = shape.N // 2

    def make(flags0):
        layers = []
        for r in range(2):
            layer = B.ExpertParallelLayer(ep_ranks=2, ep_rank=r, d_model=shape.d, n_routed=shape.N,
                                          d_ff=shape.I, n_shared=shape.Ks, d_ff_shared=shape.Is, max_tokens=300,
                                          max_k=shape.K, flags=flags0 if r == 0 else 0)
            sl = slice(r * per, (r + 1) * per)
            layer.set_weights(dev["router"], (dev["w_gate"][sl], dev["w_up"][sl], dev["w_down"][sl]),
                              (dev["ws_gate"], dev["ws_up"], dev["ws_down"]))
            layers.append(layer)
        B.connect_emulated(layers)
        return layers
    bad = make(B.MOE_FLAG_DEBUG_WAIT_TIMEOUT)
    B.forward_emulated(bad, xs, shape.K)
    assert bad[0].status() == B.MOE_ERR_TIMEOUT
    assert bad[1].status() == B.MOE_OK
    for layer in bad:
        layer.close()
    good = make(0)
    outs = B.forward_emulated(good, xs, shape.K)
    single = _single(shape, dev, None, 0, 300)
    for r in range(2):
        assert good[r].status() == B.MOE_OK
        assert torch.equal(outs[r].view(torch.int16), H.run(single, xs[r], shape.K).view(torch.int16))
