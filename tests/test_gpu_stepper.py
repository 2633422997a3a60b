"""dms_stepper_*: decode steps fed from pinned host memory, with the copies
pipelined against the kernels (through the C ABI).  Two pools get the same
prefill; one is driven by direct calls on device inputs, the other by the
stepper from packed host inputs.  The kernels and their inputs are the same,
so the outputs must agree bit for bit at every step, and the stepper's
outputs must match the fp64 oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from compact_decode_attention_b200 import dms

pytestmark = pytest.mark.gpu


def _pools_and_inputs(kind, B, Hq, Hkv, D, P, S, w, seed):
    in_kind = "f32" if kind == "f32" else "bf16"
    dt = torch.float32 if in_kind == "f32" else torch.bfloat16
    code = {"f32": dms.DMS_F32, "bf16": dms.DMS_BF16}[kind]
    K = synth.kv_tokens(seed, 0, 0, B, 0, P + S, Hkv, D, in_kind)
    V = synth.kv_tokens(seed, 1, 0, B, 0, P + S, Hkv, D, in_kind)
    fl = synth.flag_tokens(seed, 0, B, 0, P + S, Hkv, [synth.keep_threshold(0.3)] * Hkv)
    Q = np.stack([synth.q_tokens(seed, 0, B, P + s, Hq, D, in_kind) for s in range(S)])
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()  # noqa: E731
    pools = []
    for _ in range(2):
        pool = dms.Pool(1, B, Hq, Hkv, D, w, code, B * Hkv * ((P + S) // 64 + 2), P + S + 1)
        pool.compact_prefill(0, dev(K[:, :P]), dev(V[:, :P]), torch.from_numpy(fl[:, :P].copy()).cuda())
        pools.append(pool)
    return pools, K, V, fl, Q, dev, dt


@pytest.mark.parametrize("kind,B,Hq,Hkv,D", [("bf16", 3, 16, 4, 128), ("f32", 2, 8, 2, 64)])
def test_stepper_matches_direct_calls_bit_exactly(kind, B, Hq, Hkv, D):
    P, S, w = 700, 7, 64
    (pa, pb), K, V, fl, Q, dev, dt = _pools_and_inputs(kind, B, Hq, Hkv, D, P, S, w, seed=41)
    pa.set_attn_kernel(dms.ATTN_STREAM_K)   # the stepper's kernel, so the outputs can match bit for bit
    stream = torch.cuda.current_stream()
    stp = dms.Stepper(pb, 0, 1, B, stream=stream)
    hin = stp.host_inputs(S)
    hout = torch.empty(S, stp.layout.out_bytes, dtype=torch.uint8).pin_memory()
    direct = []
    for s in range(S):
        t = P + s
        k1, v1, q1 = dev(K[None, :, t]), dev(V[None, :, t]), dev(Q[None, s])
        f1 = torch.from_numpy(np.ascontiguousarray(fl[None, :, t])).cuda()
        stp.pack(hin[s], k1, v1, q1, f1)
        pa.append_evict_layers(0, t, k1, v1, f1)
        out = torch.empty(1, B, Hq, D, dtype=dt, device="cuda")
        pa.decode_attn_layers(0, q1, out)
        direct.append(out.cpu())
    for s in range(S):                      # every step enqueued before any wait
        stp.step(P + s, hin[s], hout[s])
    stp.join(stream)
    torch.cuda.synchronize()
    for s in range(S):
        got = hout[s].view(dt).view(1, B, Hq, D)
        assert torch.equal(got, direct[s]), f"step {s} differs from the direct calls"
        for b in range(B):
            exp = oatt.decode_attention(Q[s, b].astype(np.float64), K[b, :P + s + 1], V[b, :P + s + 1],
                                        fl[b, :P + s + 1], P + s, w)
            tol = 1e-5 if kind == "f32" else 2e-2
            assert np.abs(got[0, b].float().numpy() - exp).max() < tol
    stp.close()
    assert pb.stats().error_flags == 0


def test_stepper_rejects_bad_arguments():
    pool = dms.Pool(2, 2, 8, 2, 64, 16, dms.DMS_BF16, 100, 1000)
    lay = dms.dms_stepper_layout(pool.handle, 2, 2)
    assert lay.in_bytes % 256 == 0 and lay.k == 0 and lay.v % 256 == 0 and lay.evict > lay.q
    buf = torch.empty(lay.device_bytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    with pytest.raises(dms.DmsError) as e:          # device buffer too small
        dms.dms_stepper_create(pool.handle, 0, 2, 2, 0.0, buf.data_ptr(), lay.device_bytes - 256, s)
    assert e.value.status == dms.DMS_ERR_CAPACITY
    with pytest.raises(dms.DmsError) as e:          # layer range past the pool
        dms.dms_stepper_create(pool.handle, 1, 2, 2, 0.0, buf.data_ptr(), lay.device_bytes, s)
    assert e.value.status == dms.DMS_ERR_INVALID_ARG


def test_dropped_input_signal_times_out_and_the_device_keeps_answering():
    """Failure detection without a GPU fault: the stepper is told to drop one
    step's "inputs staged" signal (a lost completion message, injected on the
    host).  That step's append kernel waits for it only until the pool's wait
    limit (20 ms here instead of the default second), reports
    DMS_DEVERR_TIMEOUT and returns; dms_pool_stats then answers
    DMS_ERR_DEVICE, and later steps run on the same context as before."""
    B, Hq, Hkv, D, P, S, w = 2, 8, 2, 64, 300, 5, 32
    (pa, pb), K, V, fl, Q, dev, dt = _pools_and_inputs("bf16", B, Hq, Hkv, D, P, S, w, seed=43)
    stream = torch.cuda.current_stream()
    pb.set_wait_limit(20_000_000)
    with pytest.raises(dms.DmsError) as e:
        pb.set_wait_limit(0)
    assert e.value.status == dms.DMS_ERR_INVALID_ARG
    stp = dms.Stepper(pb, 0, 1, B, stream=stream)
    hin = stp.host_inputs(S)
    hout = torch.zeros(S, stp.layout.out_bytes, dtype=torch.uint8).pin_memory()
    for s in range(S):
        stp.pack(hin[s], dev(K[None, :, P + s]), dev(V[None, :, P + s]), dev(Q[None, s]),
                 torch.from_numpy(np.ascontiguousarray(fl[None, :, P + s])).cuda())
    for s in range(2):
        stp.step(P + s, hin[s], hout[s])
    stp.join(stream)
    torch.cuda.synchronize()
    assert pb.stats().error_flags == 0
    try:
        stp.inject_fault(dms.FAULT_DROP_INPUT_SIGNAL)
    except dms.DmsError as err:        # event protocol: nothing to drop
        assert err.status == dms.DMS_ERR_UNSUPPORTED
        stp.close()
        pytest.skip("stepper runs on events here")
    import time
    t0 = time.perf_counter()
    stp.step(P + 2, hin[2], hout[2])
    stp.join(stream)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    st = pb.stats(check=False)
    assert st.error_flags & dms.DEVERR_TIMEOUT, st.as_dict()
    with pytest.raises(dms.DmsError) as e:
        pb.stats()
    assert e.value.status == dms.DMS_ERR_DEVICE
    assert 0.015 < waited < 0.9, waited           # the 20 ms limit, not the default second
    for s in range(3, S):                         # the context still answers
        stp.step(P + s, hin[s], hout[s])
    stp.join(stream)
    torch.cuda.synchronize()
    out = hout[S - 1].view(dt).view(1, B, Hq, D).float()
    assert torch.isfinite(out).all()
    stp.close()
    assert float(torch.ones(4, device="cuda").sum().item()) == 4.0
