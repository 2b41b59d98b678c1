"""stq_prefill_chunk_noalloc: the chunked prefill with its workspace in the library's own fixed
device array. Collected last, so that it runs after every other test as well as alone.

The GPU test compares it with stq_prefill_chunk given a workspace, on two calls in a row that
continue one prompt (the second call starts from the state the first one wrote); the host test
checks the size limit, which is enforced before any device work.
"""
import pytest
import torch

DEV = "cuda"


@pytest.fixture(scope="module")
def stq():
    import quantized_linear_attention_stq_b200 as m

    m.lib()
    return m


def test_noalloc_rejects_calls_beyond_its_array(stq):
    """One chunk of the widest width class must fit the 32 MiB array: 288 requests of a single
    4-bit head need 288 records of 116736 bytes, one more than fit, and are refused before any
    device work (the fake pointers are never dereferenced)."""
    import ctypes

    bf = torch.bfloat16
    lay = stq.Layout([4, 16], 128, in_dtype=bf)
    rec = stq.prefill_workspace_bytes(stq.Layout([4], 128, in_dtype=bf), 1, 64, 64)
    assert (32 << 20) // rec == 287
    L = stq.lib()
    fake = ctypes.c_void_p(0x10000)
    args = (lay.handle, fake, 400, fake)
    tail = (64, 64, fake, fake, fake, fake, fake, fake, fake, None, None)
    assert L.stq_prefill_chunk_noalloc(*args, 288, *tail) == 2  # STQ_ERR_UNSUPPORTED
    # arguments are checked as for stq_prefill_chunk
    assert L.stq_prefill_chunk_noalloc(*args, 2, 64, 0, *tail[2:]) == 1
    assert L.stq_prefill_chunk_noalloc(*args, 0, 64, 64, *tail[2:]) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("B,T", [(2, 150), (5, 33 * 64 + 7)])
def test_noalloc_equals_workspace_form_on_two_calls_in_a_row(stq, B, T):
    """Mixed widths with an FP16 pivot; the second case needs more than one segment of records in
    both forms (34 chunks per call). Pool bytes, readouts and status agree bit for bit after each
    of two consecutive calls."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    bits = [6, 16, 4, 8, 6]
    d, C = 128, 64
    wl = wlm.scaled(wlm.WORKLOADS["prefill16_b16_6bit"], batch=B, heads=len(bits))
    lay = stq.Layout(bits, d, in_dtype=torch.bfloat16)
    w = wlm.impact_weights(wl, DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV).flip(0).contiguous()
    pool0 = lay.alloc_pool(B, DEV)
    stq.init_state(lay, pool0, slots, torch.stack([wlm.initial_state(wl, r, DEV) for r in range(B)]), w)
    pool_ws, pool_na = pool0.clone(), pool0.clone()
    ws = torch.empty(stq.prefill_workspace_bytes(lay, B, T, C), dtype=torch.uint8, device=DEV)
    st_ws = torch.zeros(1, dtype=torch.int32, device=DEV)
    st_na = torch.zeros(1, dtype=torch.int32, device=DEV)
    for call in range(2):
        inp = wlm.prefill_inputs(wl, call * T, T, DEV)
        o_ws = torch.zeros(B, len(bits), T, d, device=DEV)
        o_na = torch.full((B, len(bits), T, d), float("nan"), device=DEV)
        args = (inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], w)
        stq.prefill_chunk(lay, pool_ws, slots, *args, o_ws, chunk=C, workspace=ws, status=st_ws)
        stq.prefill_chunk_noalloc(lay, pool_na, slots, *args, o_na, chunk=C, status=st_na)
        torch.cuda.synchronize()
        assert st_ws.item() == 0 and st_na.item() == 0, (stq.status_flags(st_ws), stq.status_flags(st_na))
        assert torch.equal(pool_ws, pool_na), f"call {call}: pool bytes differ"
        assert torch.equal(o_ws, o_na), f"call {call}: readouts differ"
    assert not torch.equal(pool_ws, pool0)
