"""The block with host-resident activations (coda_rmsnorm_block_host).

Rows stream through in chunks whose copies overlap the compute; every chunk
runs the same two GEMMs on its rows, so the output must equal, bit for bit,
the device-resident two-launch block on the whole batch (and so the fp64
oracle within the usual bar, which the other block tests establish).
"""
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


@pytest.mark.parametrize("shape,chunk,with_res", [((256, 512, 512, 1536), 256, True),
                                                  ((1000, 264, 776, 392), 256, True),
                                                  ((1000, 264, 776, 392), 512, False),
                                                  ((8192, 2048, 2048, 16384), 1024, True)])
def test_host_block_equals_device_block(shape, chunk, with_res):
    M, K, N, N2 = shape
    inp = synth.tiny_block() if shape == (256, 512, 512, 1536) else \
        synth.llama1b_block_tail(with_down=False) if M == 8192 else \
        synth.block_inputs(M, K, N, N2, seed=60 + chunk, w_std=0.04)
    W1, W2, gamma = (t.cuda() for t in (inp.W1, inp.W2, inp.gamma))
    x_h = inp.x.pin_memory()
    res_h = inp.res.pin_memory() if with_res else None
    out_h = C.rmsnorm_block_host(x_h, res_h, W1, W2, gamma, inp.eps, chunk_rows=chunk)
    again = C.rmsnorm_block_host(x_h, res_h, W1, W2, gamma, inp.eps, chunk_rows=chunk)
    torch.cuda.synchronize()
    C.poll_status()
    ref = C.gemm_rmsnorm_gemm(inp.x.cuda(), None if res_h is None else inp.res.cuda(), W1, W2, gamma, inp.eps)
    torch.cuda.synchronize()
    assert torch.equal(out_h, ref["out"].cpu())
    assert torch.equal(again, out_h)


def test_host_block_rejects_device_tensors_and_bad_chunks():
    inp = synth.tiny_block()
    W1, W2, gamma = (t.cuda() for t in (inp.W1, inp.W2, inp.gamma))
    with pytest.raises(ValueError):
        C.rmsnorm_block_host(inp.x.cuda(), None, W1, W2, gamma, inp.eps)
    with pytest.raises(C.CodaError):
        C.rmsnorm_block_host(inp.x.pin_memory(), None, W1, W2, gamma, inp.eps, chunk_rows=100)


def test_host_block_concurrent_callers():
    """Two host threads, each on its own stream and workspace, call the
    host-buffer block at the same time: the library's shared copy streams
    and events must keep every call's copies ordered after its own compute."""
    import threading

    shape = (1000, 264, 776, 392)
    M, K, N, N2 = shape
    ins = [synth.block_inputs(M, K, N, N2, seed=70 + t, w_std=0.04) for t in range(2)]
    W1, W2, gamma = (t.cuda() for t in (ins[0].W1, ins[0].W2, ins[0].gamma))
    refs = [C.gemm_rmsnorm_gemm(i.x.cuda(), i.res.cuda(), W1, W2, gamma, i.eps)["out"].cpu() for i in ins]
    nb = int(C.load_library().coda_rmsnorm_block_host_workspace_size(K, N, N2, 256))
    outs = [[], []]
    errors = []

    def worker(t):
        try:
            s = torch.cuda.Stream()
            ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
            x_h, res_h = ins[t].x.pin_memory(), ins[t].res.pin_memory()
            with torch.cuda.stream(s):
                for _ in range(24):
                    outs[t].append(C.rmsnorm_block_host(x_h, res_h, W1, W2, gamma, ins[t].eps, chunk_rows=256, ws=ws))
            s.synchronize()
        except Exception as e:  # reported on the main thread
            errors.append(e)

    th = [threading.Thread(target=worker, args=(t,)) for t in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
    C.poll_status()
    for t in range(2):
        assert len(outs[t]) == 24
        for o in outs[t]:
            assert torch.equal(o, refs[t])
