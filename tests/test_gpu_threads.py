"""Several host threads calling the entry points at once, each on its own CUDA
stream (the library's per-device launch caches are shared between them):
every call returns the bytes a single-threaded call returns."""
import threading

import pytest
import torch

from mixture_experts_routed_expert_b200 import inputs

pytestmark = pytest.mark.gpu


def test_concurrent_host_threads(cuda_dev):
    import mixture_experts_routed_expert_b200 as moe
    base = inputs.ocr2_layer(1, seed=0, device=cuda_dev)
    cases = [(T, fn) for T in (1, 2, 64, 300)
             for fn in ("moe_experts_decode", "moe_experts_prefill")]
    lays = {T: inputs.ocr2_layer(T, seed=40 + T, device=cuda_dev, weights_from=base)
            for T in {T for T, _ in cases}}

    def call(T, fn):
        lay = lays[T]
        return getattr(moe, fn)(lay.x, lay.gate_up, lay.down, lay.idx, lay.w, lay.idx.shape[1])

    ref = {c: call(*c) for c in cases}
    torch.cuda.synchronize()
    got, errors = {}, []
    start = threading.Barrier(len(cases))

    def worker(case):
        try:
            with torch.cuda.device(cuda_dev):
                stream = torch.cuda.Stream()
                with torch.cuda.stream(stream):
                    start.wait()
                    for _ in range(5):
                        got[case] = call(*case)
                stream.synchronize()
        except Exception as exc:   # reported on the main thread
            errors.append((case, exc))

    threads = [threading.Thread(target=worker, args=(c,)) for c in cases]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads), "a caller thread did not finish"
    assert not errors, errors
    torch.cuda.synchronize()
    for c in cases:
        assert torch.equal(got[c], ref[c]), "T=%d %s differs under concurrent callers" % c
