"""csa_sparse_attend_noalloc: the attention entry point for callers that may
not allocate device memory (for instance a plug-in inside a host framework
that owns every device allocation, or a serving loop that must never enter
the driver's allocator).  It must give what csa_sparse_attend gives with a
workspace, call after call, using only the library's fixed device scratch.

This file is collected last on purpose: the first call on a device sets up
the scratch address, and the test must pass both alone in a fresh process
and after every other test."""
import numpy as np
import pytest
import torch

from long_context_sparse_03_b200 import csa
from tests.gpu_cases import check_attention, dev_bf16, dev_i32, host_bits
from tests.pins import bf16_bits_to_f64, rand_bf16

pytestmark = pytest.mark.gpu


def _case(rng, T, H, k, W, m=4, B=3, N=3000):
    L = N * m + 5
    q = rand_bf16(rng, (T, H, 128))
    comp = rand_bf16(rng, (B, N, 128))
    raw = rand_bf16(rng, (B, L, 128))
    q_seq = rng.integers(0, B, T).astype(np.int32)
    q_pos = rng.integers(0, N * m, T).astype(np.int32)
    q_pos[0] = N * m - 1
    idx = np.full((T, k), -1, np.int32)
    for t in range(T):
        V = (q_pos[t] + 1) // m
        n = min(k, V)
        if n:
            idx[t, :n] = rng.choice(V, n, replace=False)
    return [dev_bf16(q), dev_i32(q_seq), dev_i32(q_pos), dev_bf16(comp), dev_bf16(raw), m, dev_i32(idx), W]


def test_noalloc_matches_workspace_entry_twice():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    rng = np.random.default_rng(2024)
    scale = 128 ** -0.5
    for T, H, k, W in ((8, 64, 1024, 128), (5, 16, 300, 37)):
        q, q_seq, q_pos, comp, raw, m, idx, Wd = _case(rng, T, H, k, W)
        ref = torch.empty((T, H, 128), dtype=torch.bfloat16, device="cuda")
        ref_lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
        ws = csa.Workspace(csa.csa_attend_workspace_size(T, H, k + W))
        csa.csa_sparse_attend(q, q_seq, q_pos, comp, raw, m, idx, Wd, scale, ref, ref_lse, ws)
        torch.cuda.synchronize()
        r = bf16_bits_to_f64(host_bits(ref))
        rl = ref_lse.cpu().numpy().astype(np.float64)
        for _ in range(2):   # two calls in a row share the same scratch
            out = torch.full((T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
            lse = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
            csa.csa_sparse_attend_noalloc(q, q_seq, q_pos, comp, raw, m, idx, Wd, scale, out, lse)
            torch.cuda.synchronize()
            check_attention(bf16_bits_to_f64(host_bits(out)), lse.cpu().numpy().astype(np.float64), r, rl)


def test_noalloc_rejects_oversized_call():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    rng = np.random.default_rng(7)
    T, H, k, W = 64, 128, 2048, 1024          # far beyond the fixed scratch
    q, q_seq, q_pos, comp, raw, m, idx, Wd = _case(rng, T, H, k, W, N=600)
    assert csa.csa_attend_workspace_size(T, H, k + W) > csa.NOALLOC_SCRATCH_BYTES
    out = torch.empty((T, H, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(csa.CsaError) as e:
        csa.csa_sparse_attend_noalloc(q, q_seq, q_pos, comp, raw, m, idx, Wd, 0.1, out, None)
    assert e.value.status == 4
