"""The failure path of the kernels' bounded waits, driven on the GPU without
faulting or hanging it: sage_wait_probe launches one CTA whose mbarrier wait
is never satisfied and gives up after a short limit. The test checks that the
probe returns, that the error word reaches the host as SAGE_ERR_TIMEOUT with
the probe's kernel id and wait site, that reading it clears it, and that the
device is still usable: a following quantised attention call matches the
oracle."""
import time

import pytest
import torch

import oracle
import quantized_attention_smoothing_b200 as sage
import workloads
from gpu_helpers import bits, compare_output, to_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib_built():
    from quantized_attention_smoothing_b200 import build
    build.build()
    return sage.lib()


def test_wait_probe_times_out_and_device_stays_usable(lib_built):
    torch.cuda.set_device(0)
    assert sage.sage_device_error_where()[0] == sage.SAGE_OK       # nothing pending
    t0 = time.perf_counter()
    sage.sage_wait_probe(10_000_000)                                # 10 ms limit
    st, kernel, site = sage.sage_device_error_where()               # synchronises
    elapsed = time.perf_counter() - t0
    assert st == sage.SAGE_ERR_TIMEOUT
    assert kernel == sage.SAGE_KERNEL_PROBE and site == 1
    # the second waiter ended through the abort flag, well before its own 2 s
    assert elapsed < 1.5, elapsed
    assert sage.sage_device_error_where() == (sage.SAGE_OK, 0, 0)  # read and cleared

    cfg, q, k, v = workloads.make_prefill_config("c1")
    h = sage.Hadamard(cfg["D"])
    out, _ = sage.sage_attention(h, to_gpu(q), to_gpu(k), to_gpu(v), cfg["blk_q"], cfg["blk_k"],
                                 cfg["softmax_scale"], cfg["causal"])
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    qk = oracle.quant_qk(bits(q), bits(k), cfg["blk_q"], cfg["blk_k"])
    v8t, vs = oracle.quant_v(bits(v))
    _, ref = oracle.attn(qk["q8"], qk["qs"], qk["k8"], qk["ks"], v8t, vs, cfg["L"], cfg["L"],
                         cfg["blk_q"], cfg["blk_k"], cfg["softmax_scale"], cfg["causal"],
                         want_f64=True)
    compare_output(bits(out), ref, None, label="after the probe")


def test_wait_probe_rejects_out_of_range_limits(lib_built):
    for bad in (0, 999, 10_000_000_001):
        with pytest.raises(sage.SageError) as e:
            sage.sage_wait_probe(bad)
        assert e.value.status == sage.SAGE_ERR_INVALID_ARG
