"""Expert parallelism on one GPU: G ranks simulated by G threads that share
the device and exchange rows through an in-process all-to-all; each rank
holds its own tokens and E/G of the experts and runs ep_forward with the
library's kernels (moe_experts_rows for its experts, moe_combine_rows for
its tokens).  Every rank's output must equal moe_experts_prefill of the
same tokens with all experts, bit for bit (each row is computed by the same
kernels and summed in the same order, whatever the sharding), and match the
oracle."""
import threading

import pytest
import torch

import oracle
from _helpers import assert_matches_oracle
from mixture_experts_routed_expert_b200 import inputs
from mixture_experts_routed_expert_b200.ep import ep_forward

pytestmark = pytest.mark.gpu


class ThreadExchange:
    """all-to-all between G threads of one process (one per simulated rank)."""

    def __init__(self, world):
        self.world = world
        self.barrier = threading.Barrier(world, timeout=120)
        self.box = {}

    def rank_view(self, rank):
        ex = self

        class View:
            world = ex.world

            def __init__(self):
                self.rank = rank
                self.seq = 0

            def _swap(self, parts):
                key = self.seq
                self.seq += 1
                ex.box[(key, self.rank)] = parts
                ex.barrier.wait()
                got = [ex.box[(key, j)][self.rank] for j in range(ex.world)]
                ex.barrier.wait()
                return got

            def counts(self, send_counts):
                got = self._swap(list(send_counts.split(1)))
                return torch.cat(got)

            def rows(self, send, send_splits, recv_splits):
                got = self._swap(list(send.split(send_splits)))
                assert [g.shape[0] for g in got] == list(recv_splits)
                return torch.cat(got).contiguous()
        return View()


@pytest.mark.parametrize("world,T,E,skew", [(2, 37, 64, None), (4, 200, 64, 1.1), (2, 1, 64, None)])
def test_ep_matches_single_gpu(cuda_dev, world, T, E, skew):
    import mixture_experts_routed_expert_b200 as moe
    H, F, K = 1280, 896, 6
    full = inputs.ocr2_layer(1, seed=3, device=cuda_dev)
    lays = [inputs.ocr2_layer(T + r, seed=70 + r, device=cuda_dev, weights_from=full, zipf=skew)
            for r in range(world)]
    lays[0].idx[0, 2] = -1                          # a slot that is not sent
    ex = ThreadExchange(world)
    El = E // world
    outs, errs = [None] * world, []

    def run(r):
        try:
            mine = slice(r * El, (r + 1) * El)
            outs[r] = ep_forward(lays[r].x, full.gate_up[mine], full.down[mine], lays[r].idx,
                                 lays[r].w, E, exchange=ex.rank_view(r))
        except Exception as e:   # reported below
            errs.append(e)
            ex.barrier.abort()
    th = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=300)
    assert not errs, errs
    torch.cuda.synchronize()
    for r in range(world):
        ref = moe.moe_experts_prefill(lays[r].x, full.gate_up, full.down, lays[r].idx, lays[r].w, K)
        assert torch.equal(outs[r].view(torch.int16), ref.view(torch.int16)), r
    tk = torch.arange(min(8, T))
    lay = lays[-1]
    o = oracle.moe_forward_bf16(inputs.bf16_bits(lay.x.cpu()[tk]), inputs.bf16_bits(full.gate_up),
                                inputs.bf16_bits(full.down), inputs.np32(lay.idx.cpu()[tk]),
                                inputs.np32(lay.w.cpu()[tk]))
    assert_matches_oracle(outs[-1][tk.to(cuda_dev)], o, "ep world=%d" % world)
