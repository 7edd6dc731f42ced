"""The continuous-batching step as a CUDA graph: the uploads and the append +
decode launches captured once per staging set and replayed, bit for bit equal
to the same steps run eagerly (same fixed decode plan), for the fused and the
two-call step; the replayed output also against the oracle on sampled
(request, head) pairs of the last step."""

import types

import numpy as np
import pytest
import torch

from helpers import assert_parity, oracle_pairs
from paged_kv_cache_driven_b200 import binding, workloads
from paged_kv_cache_driven_b200.batching import ContinuousBatching

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "two_calls"])
def test_graph_replay_equals_eager(fused):
    steps = 24
    runs = {}
    for graph in (False, True):
        loop = workloads.batching_loop(seed=5, batch=16, H=4)
        cb = ContinuousBatching(loop, DEV, max_steps=steps, fused=fused, graph=graph,
                                fixed_plan=True)
        outs, recs = [], []
        for k in range(steps):
            rec = cb.step(k)
            outs.append(cb.out.clone())
            recs.append(rec)
        torch.cuda.synchronize()
        assert binding.pa_get_device_error() == 0
        runs[graph] = (cb, outs, recs)
    cb_e, outs_e, recs_e = runs[False]
    cb_g, outs_g, recs_g = runs[True]
    assert all(g is not None for g in cb_g.graphs)
    for k in range(steps):
        assert recs_e[k]["ids"] == recs_g[k]["ids"]
        assert torch.equal(recs_e[k]["tables"], recs_g[k]["tables"])
        assert torch.equal(outs_e[k], outs_g[k]), f"step {k}"
    assert torch.equal(bits(cb_e.k_cache), bits(cb_g.k_cache))
    assert torch.equal(bits(cb_e.v_cache), bits(cb_g.v_cache))
    assert cb_e.alloc.pa_alloc_dump() == cb_g.alloc.pa_alloc_dump()
    # the last replayed step against the oracle
    rec = recs_g[-1]
    S = cb_g.S
    lens = rec["lens"].tolist()
    case = types.SimpleNamespace(
        q=rec["q"], k_cache=cb_g.k_cache, v_cache=cb_g.v_cache, seq_lens_host=lens, scale=cb_g.scale,
        tables_host=[rec["tables"][i, : -(-L // S)].tolist() for i, L in enumerate(lens)])
    # requests that retired after the step may have had their blocks reused
    live = [i for i, sid in enumerate(rec["ids"]) if sid not in rec["retired"]]
    pairs = [(i, h) for i in live[::3] for h in range(4)]
    want = oracle_pairs(case, pairs)
    got = torch.stack([outs_g[-1][i, h] for i, h in pairs]).cpu().numpy()
    assert_parity(got, want, "replayed step vs oracle")
