"""Expert parallelism on CPU (gloo, world size 2): the dispatch plan against
a brute-force restatement, and the whole dispatch -> experts -> return ->
combine exchange against the same per-row computation done on one rank (the
row function here is the oracle's forward of one slot, so that only the
exchange is under test: the result must not depend on the sharding, bit for
bit)."""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from mixture_experts_routed_expert_b200 import inputs
from mixture_experts_routed_expert_b200.ep import ep_forward, ep_plan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _plan_brute(idx, E, world):
    El = E // world
    T, K = idx.shape
    slots = [(t * K + k, int(idx[t, k])) for t in range(T) for k in range(K)
             if 0 <= int(idx[t, k]) < E]
    order = [s for r in range(world) for s, e in slots if e // El == r]
    counts = [sum(1 for _, e in slots if e // El == r) for r in range(world)]
    local = [int(idx.reshape(-1)[s]) - (int(idx.reshape(-1)[s]) // El) * El for s in order]
    return order, counts, local


@pytest.mark.parametrize("T,K,E,world,seed", [(5, 3, 8, 2, 0), (16, 6, 64, 4, 1), (1, 8, 16, 8, 2),
                                              (9, 2, 4, 1, 3)])
def test_plan_matches_brute_force(T, K, E, world, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.randint(-2, E + 2, (T, K), generator=g, dtype=torch.int32)
    order, counts, local = ep_plan(idx, E, world)
    bo, bc, bl = _plan_brute(idx.numpy(), E, world)
    assert order.tolist() == bo and counts.tolist() == bc and local.tolist() == bl
    with pytest.raises(ValueError):
        ep_plan(idx, E + 1, 2) if (E + 1) % 2 else ep_plan(idx, E, 3)


def _rows_oracle(gate_up, down):
    """y rows (fp32) of single slots: the oracle's forward with one slot of
    weight w, read back from its bf16 output."""
    gu, dn = inputs.bf16_bits(gate_up), inputs.bf16_bits(down)

    def fn(x, ids, w):
        if x.shape[0] == 0:
            return torch.zeros(0, x.shape[1], dtype=torch.float32)
        o = oracle.moe_forward_bf16(inputs.bf16_bits(x), gu, dn, inputs.np32(ids), inputs.np32(w))
        return torch.from_numpy(oracle.bf16_to_f64(o).astype(np.float32))
    return fn


def _combine_k_order(y, idx, E):
    T, K = idx.shape
    acc = torch.zeros(T, y.shape[1], dtype=torch.float32)
    for k in range(K):
        v = ((idx[:, k] >= 0) & (idx[:, k] < E)).unsqueeze(1)
        acc = acc + torch.where(v, y.view(T, K, -1)[:, k], torch.zeros_like(acc))
    return acc.to(torch.bfloat16)


def _worker(rank, world, port, result_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, H, F, E, K = 7 + rank, 128, 128, 8, 3
        full = inputs.ocr2_layer(1, seed=5, H=H, F=F, E=E, K=K)        # every rank: same weights
        lay = inputs.ocr2_layer(T, seed=40 + rank, H=H, F=F, E=E, K=K, weights_from=full)
        idx = lay.idx.clone()
        idx[0, 1] = -1                                                   # a slot that is not sent
        El = E // world
        mine = slice(rank * El, (rank + 1) * El)
        out = ep_forward(lay.x, full.gate_up[mine], full.down[mine], idx, lay.w, E,
                         rows_fn=_rows_oracle(full.gate_up[mine], full.down[mine]),
                         combine_fn=lambda y, i: _combine_k_order(y, i, E))
        # the same rows computed on one rank, slot by slot with global ids
        rows = _rows_oracle(full.gate_up, full.down)
        flat = idx.reshape(-1)
        valid = (flat >= 0) & (flat < E)
        y = torch.zeros(T * K, H, dtype=torch.float32)
        sl = torch.nonzero(valid).reshape(-1)
        y[sl] = rows(lay.x[sl // K], flat[sl].view(-1, 1), lay.w.reshape(-1)[sl].view(-1, 1))
        ref = _combine_k_order(y, idx, E)
        ok = torch.equal(out.view(torch.int16), ref.view(torch.int16))
        open(os.path.join(result_dir, "r%d" % rank), "w").write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_exchange_is_sharding_independent(tmp_path):
    world = 2
    port = 29600 + (os.getpid() % 200)
    mp.spawn(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        assert open(tmp_path / ("r%d" % r)).read() == "ok", r
