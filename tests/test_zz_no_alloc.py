"""GPU test of cca_chunk_attn_noalloc, the allocation-free attention entry point.

It exists for callers that cannot give the library device scratch memory (a
running real-time stream loop that must not call the device allocator, or a
host application that owns all device memory and offers plug-ins no
allocator).  Its scratch is an array built into libcca.so and shared by all
calls.  The test calls it through the C ABI twice in a row (so the second call
starts from the first call's leftover scratch) and compares each result with the
allocating entry point cca_chunk_attn bit for bit: both run the same kernels
with the same grid and schedule, only the scratch address differs, so any
difference (a stale partial result left in the shared array, say) is a bug.
It also checks that a call needing more scratch than the array holds is
refused with a message.  This file is collected last on purpose.
"""

import pytest
import torch

import chunk_causal_attention_b200 as cca
import synth

pytestmark = pytest.mark.gpu


def _noalloc(ring, q, k, v, out, n_q_max):
    L = cca.lib()
    return L.cca_chunk_attn_noalloc(ring.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), None, None, None,
                                    None, None, int(n_q_max), 0.0, out.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_allocating_entry_point_on_two_calls(monkeypatch):
    dev = torch.device("cuda:0")
    monkeypatch.delenv("CCA_ATTN_CTAS", raising=False)  # default grid: 20 of 168 items are split
    c1 = synth.chunk_720p()
    ring = cca.KVRing(c1.n_heads, c1.head_dim, c1.chunk_len, c1.window, device=dev)
    for t in range(c1.t):
        ring.append(synth.as_torch_bf16(c1.ring_k[t], dev), synth.as_torch_bf16(c1.ring_v[t], dev))
    assert cca.cca_chunk_attn_workspace_size(ring, c1.chunk_len) > 0
    for s in range(2):  # two calls in a row, different inputs
        q = synth.as_torch_bf16(c1.q[s], dev)
        k = synth.as_torch_bf16(c1.k_cur[s], dev)
        v = synth.as_torch_bf16(c1.v_cur[s], dev)
        ref = cca.cca_chunk_attn(ring, q, k, v)
        out = torch.full_like(ref, float("nan"))
        st = _noalloc(ring, q, k, v, out, c1.chunk_len)
        assert st == 0, cca.lib().cca_last_error().decode()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {s}: {(out.float() - ref.float()).abs().max().item()}"
    assert int(ring.status.item()) == 0


def test_noalloc_refuses_calls_beyond_its_scratch(monkeypatch):
    dev = torch.device("cuda:0")
    monkeypatch.setenv("CCA_ATTN_CTAS", "400")  # 2 x 400 slots x 256 rows x 130 x 4 B > 64 MiB
    c1 = synth.chunk_720p(n_steps=1, n_prefill=1)
    ring = cca.KVRing(c1.n_heads, c1.head_dim, c1.chunk_len, c1.window, device=dev)
    ring.append(synth.as_torch_bf16(c1.ring_k[0], dev), synth.as_torch_bf16(c1.ring_v[0], dev))
    q = synth.as_torch_bf16(c1.q[0], dev)
    out = torch.empty((c1.chunk_len, c1.n_heads, c1.head_dim), dtype=torch.bfloat16, device=dev)
    st = _noalloc(ring, q, q, q, out, c1.chunk_len)
    assert st == 1  # CCA_ERR_INVALID_ARG
    assert "scratch" in cca.lib().cca_last_error().decode()
