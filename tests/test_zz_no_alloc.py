"""mtla_decode_attn_static (scratch in a static device array, no workspace)
against mtla_decode_attn with a caller workspace, through the C ABI.

The file name sorts last, so the test also runs after every other GPU test has
used the library in the same process; it must pass alone as well."""
import numpy as np
import pytest
import torch

import mtla_synth as synth
import temporally_compressed_latent_b200 as mtla
from gpu_harness import DecodeRun, assert_close, dev, host, oracle_decode

pytestmark = pytest.mark.gpu


def _static_step(run: DecodeRun, q_abs, q_rope, c_new=None, kR_new=None):
    merge = None
    if c_new is not None:
        run._c = dev(c_new, run.dtype)
        run._k = dev(kR_new, run.dtype)
        merge = {"c_new": run._c, "kR_new": run._k, "W_c": run.W_c, "b_c": run.b_c, "P": run.P,
                 "J_max": run.J_max}
    run._qa = dev(q_abs, run.dtype)
    run._qr = dev(q_rope, run.dtype)
    torch.cuda.synchronize()
    # the inputs are on the device: from here on nothing may take device memory
    run.free_before_call = torch.cuda.mem_get_info()[0]
    mtla.mtla_decode_attn_static(run.md, run.B, run._qa, run._qr, merge, run.cache.buf, run.cache.cache_rows,
                                 run.cache.row_stride, run.cache.offset, run.cache.capacity, run.t, run.cache_len,
                                 run.out, run.lse, run.err)
    torch.cuda.synchronize()
    return host(run.out), host(run.lse)


def test_static_scratch_matches_workspace_entry():
    """Two consecutive merge steps and one read-only call, on the split-L
    tensor-core path (bf16, H=8, r=256, d_R=32): same outputs, lengths and
    cache as the workspace entry on an identical copy of the state."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    rng = np.random.default_rng(61)
    t_prev = np.concatenate([[1, 2, 127, 128, 4095, 4096], rng.integers(1, 3000, size=42)])
    case = synth.decode_case(dims, t_prev, seed=62, dtype="bf16")
    ref = DecodeRun(case)
    sta = DecodeRun(case)
    assert ref.ws_bytes > 0, "this case must use the scratch-using tensor-core kernel"
    # every B the tensor-core path accepts fits the static scratch on this device
    assert mtla.mtla_workspace_bytes(ref.md, 1024) <= mtla.DECODE_STATIC_SCRATCH_BYTES

    rows = [list(np.asarray(r, np.float64)) for r in case.rows]
    t_prev = case.t_prev.copy()
    for step in range(2):
        qa = synth.cast(rng.standard_normal((case.B, 8, 256)), "bf16")
        qr = synth.cast(rng.standard_normal((case.B, 8, 32)), "bf16")
        cn = synth.cast(rng.standard_normal((case.B, 256)), "bf16")
        kn = synth.cast(rng.standard_normal((case.B, 32)), "bf16")
        o_ref, l_ref = ref.step(qa, qr, cn, kn)
        o_sta, l_sta = _static_step(sta, qa, qr, cn, kn)
        if step > 0:
            # after the set-up of the first call (which may load the array: the
            # driver reserves it when it loads the library's device code, at
            # first use under lazy loading), a call takes no device memory
            assert torch.cuda.mem_get_info()[0] == sta.free_before_call
        assert_close(o_sta, o_ref, "bf16", f"step {step} out")
        assert_close(l_sta, l_ref, "bf16", f"step {step} lse")
        # and both against the fp64 oracle stepping the same tokens
        o_orc, l_orc, r_orc = oracle_decode(case, ref.J_max, q_abs=qa, q_rope=qr, c_new=cn, kR_new=kn, rows=rows,
                                            t_prev=t_prev)
        assert_close(o_sta, np.stack([o_orc[b] for b in range(case.B)]), "bf16", f"step {step} out vs oracle")
        assert_close(l_sta, np.stack([l_orc[b] for b in range(case.B)]), "bf16", f"step {step} lse vs oracle")
        # the oracle continues from the device's bf16 cache rows
        rows = [list(sta.cache.rows(b, len(r_orc[b]))) for b in range(case.B)]
        t_prev = t_prev + 1
        assert sta.t.cpu().tolist() == ref.t.cpu().tolist()
        assert sta.cache_len.cpu().tolist() == ref.cache_len.cpu().tolist()
        assert int(sta.err.item()) == 0 and int(ref.err.item()) == 0
    for b in range(case.B):
        L = int(ref.cache_len[b].item())
        assert_close(sta.cache.rows(b, L), ref.cache.rows(b, L), "bf16", f"cache b={b}")

    # a read-only call (no merge) on the state the two steps left
    o_ref, l_ref = ref.step(case.q_abs, case.q_rope)
    o_sta, l_sta = _static_step(sta, case.q_abs, case.q_rope)
    assert_close(o_sta, o_ref, "bf16", "read-only out")
    assert_close(l_sta, l_ref, "bf16", "read-only lse")
