"""Parity at the full workload sizes, in the launch configuration bench.py
times, on sampled sequences the oracle can afford.

Each workload is drawn at full size on the device from its seed.  For a few
sampled sequences the raw rows are copied to the host and the oracle builds
its own caches; those caches replace the GPU's for the sampled sequences,
and the GPU stages (indexer select, attention) run over the whole batch in
the bench's launch configuration.  The sampled queries are then judged
stage-wise against the oracle (tolerances: tests/gpu_cases.py), and the
GPU's own caches for those sequences against the oracle's.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_03_b200 import csa
from long_context_sparse_03_b200 import workloads as wl
from tests.gpu_cases import check_attention, check_compress_bf16, check_topk, host_bits, score_scale
from tests.pins import bf16_bits_to_f64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    csa.lib()


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _csa_decode(oracle, w, samples, fmt):
    inp = wl.make_inputs(w, device="cuda")
    B, N, T = w.B, w.max_blocks, w.B
    comp = torch.empty((B, N, 128), dtype=torch.bfloat16, device="cuda")
    if fmt == 0:
        kid = torch.empty((B, N, 64), dtype=torch.bfloat16, device="cuda")
        ksc = None
    else:
        kid = torch.empty((B, N, 64), dtype=torch.uint8, device="cuda")
        ksc = torch.empty((B, N), dtype=torch.float32, device="cuda")
    csa.csa_compress(inp.raw_kv, inp.lens, inp.z_kv, w.m, 0, N, comp)
    csa.csa_compress(inp.raw_ki, inp.lens, inp.z_ki, w.m, 0, N, kid, fmt, ksc)
    torch.cuda.synchronize()
    lens = inp.lens.cpu().numpy()
    z_kv, z_ki = inp.z_kv.cpu().numpy(), inp.z_ki.cpu().numpy()
    a_kv, a_ki = oracle.pool_weights(z_kv), oracle.pool_weights(z_ki)
    ref = {}
    for b in samples:
        L = int(lens[b])
        raw_kv = _bits(inp.raw_kv[b:b + 1, :L])
        raw_ki = _bits(inp.raw_ki[b:b + 1, :L])
        ck, _ = oracle.compress(raw_kv, lens[b:b + 1], z_kv, 0, 1 << 30)
        kk, ks = oracle.compress(raw_ki, lens[b:b + 1], z_ki, 0, 1 << 30, out_fmt=fmt)
        nb = L // w.m
        # the GPU's caches of the sampled sequence against the oracle's
        sel = np.random.default_rng(b).choice(nb, min(nb, 4096), replace=False)
        gk = _bits(comp[b, :nb])[sel]
        x = bf16_bits_to_f64(raw_kv[0, :nb * w.m]).reshape(nb, w.m, 128)[sel]
        check_compress_bf16(gk, ck[0, :nb][sel], absum=np.einsum("jid,id->jd", np.abs(x), np.abs(a_kv)), m=w.m)
        if fmt == 0:
            gi = _bits(kid[b, :nb])[sel]
            xi = bf16_bits_to_f64(raw_ki[0, :nb * w.m]).reshape(nb, w.m, 64)[sel]
            check_compress_bf16(gi, kk[0, :nb][sel], absum=np.einsum("jid,id->jd", np.abs(xi), np.abs(a_ki)), m=w.m)
        else:
            gc = kid[b, :nb].cpu().numpy()[sel]
            gs = ksc[b, :nb].cpu().numpy()[sel]
            rs = ks[0, :nb][sel]
            assert (np.abs(gs - rs) / rs <= 2 ** -7).all()
            same = gs == rs
            dc = np.abs(gc.astype(np.int32) - kk[0, :nb][sel].astype(np.int32))
            assert (dc[same] <= 1).all()
        # the oracle's caches replace the GPU's for this sequence
        comp[b, :nb] = _to_dev(ck[0, :nb])
        if fmt == 0:
            kid[b, :nb] = _to_dev(kk[0, :nb])
        else:
            kid[b, :nb] = torch.from_numpy(kk[0, :nb]).cuda()
            ksc[b, :nb] = torch.from_numpy(ks[0, :nb]).cuda()
        ref[b] = (raw_kv, ck, kk, ks)
    # indexer query: GPU projection vs oracle (all queries), then the oracle's
    # q, w (as fp32) drive the selection stage
    h, Wdq, Wuq, Ww = (_bits(x) for x in (inp.h, inp.W_dq, inp.W_uq, inp.W_w))
    rq, rw = oracle.index_query(h, Wdq, Wuq, Ww)
    qg = torch.empty((T, w.Hi, 64), dtype=torch.float32, device="cuda")
    wg = torch.empty((T, w.Hi), dtype=torch.float32, device="cuda")
    ws = csa.Workspace(csa.csa_index_workspace_size(T, w.r, w.Hi, w.k, N))
    csa.csa_index_query(inp.h, inp.W_dq, inp.W_uq, inp.W_w, qg, wg, ws)
    gq, gw = qg.cpu().numpy().astype(np.float64), wg.cpu().numpy().astype(np.float64)
    for t in range(T):
        assert np.abs(gq[t] - rq[t]).max() <= 1e-5 * np.abs(rq[t]).max()
        assert np.abs(gw[t] - rw[t]).max() <= 1e-5 * np.abs(rw[t]).max()
    q32, w32 = rq.astype(np.float32), rw.astype(np.float32)
    idx = torch.empty((T, w.k), dtype=torch.int32, device="cuda")
    sc = torch.empty((T, w.k), dtype=torch.float32, device="cuda")
    csa.csa_index_select(torch.from_numpy(q32).cuda(), torch.from_numpy(w32).cuda(), inp.q_seq, inp.q_pos, kid, w.m, N,
                         w.k, idx, sc, ws, kidx_scale=ksc)
    ws.check()
    gi, gs = idx.cpu().numpy(), sc.cpu().numpy()
    q_pos = inp.q_pos.cpu().numpy()
    oidx = gi.copy()
    for b in samples:
        raw_kv, ck, kk, ks = ref[b]
        S = oracle.index_scores(q32[b:b + 1].astype(np.float64), w32[b:b + 1].astype(np.float64), [0],
                                q_pos[b:b + 1], kk, w.m, N, kidx_fmt=fmt, kidx_scale=ks)
        kf = bf16_bits_to_f64(kk[0]) if fmt == 0 else oracle.e4m3_decode(kk[0]) * ks[0][:, None].astype(np.float64)
        A = score_scale(q32[b].astype(np.float64), w32[b].astype(np.float64), kf)
        V = min((int(q_pos[b]) + 1) // w.m, N)
        check_topk(gi[b], gs[b], S[0], A, V, w.k)
        oi, _ = oracle.topk(S, q_pos[b:b + 1], w.m, w.k)
        oidx[b] = oi[0]
    # attention over the oracle's selection, whole batch in one call
    out = torch.empty((T, w.H, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
    wa = csa.Workspace(csa.csa_attend_workspace_size(T, w.H, w.k + w.W))
    csa.csa_sparse_attend(inp.q, inp.q_seq, inp.q_pos, comp, inp.raw_kv, w.m, torch.from_numpy(oidx).cuda(), w.W,
                          128 ** -0.5, out, lse, wa)
    wa.check()
    qa = _bits(inp.q)
    for b in samples:
        raw_kv, ck, kk, ks = ref[b]
        ro, rl = oracle.sparse_attend(qa[b:b + 1], [0], q_pos[b:b + 1], ck, raw_kv, w.m, oidx[b:b + 1], w.W,
                                      128 ** -0.5)
        check_attention(bf16_bits_to_f64(host_bits(out[b:b + 1])), lse[b:b + 1].cpu().numpy().astype(np.float64),
                        ro, rl)
    del inp, comp, kid, ksc
    torch.cuda.empty_cache()


@pytest.mark.parametrize("fmt", [0, 1], ids=["bf16_keys", "e4m3_keys"])
def test_csa_decode_1m_b8(oracle, fmt):
    _csa_decode(oracle, wl.CSA_DECODE_1M, samples=[0, 5], fmt=fmt)


def test_csa_decode_ragged_b32(oracle):
    _csa_decode(oracle, wl.CSA_DECODE_64K_RAGGED, samples=[0, 13, 31], fmt=0)


def test_csa_decode_4k_b1(oracle):
    w = wl.scaled(wl.CSA_DECODE_4K, device_rng=True)
    _csa_decode(oracle, w, samples=[0], fmt=0)


def test_hca_decode_1m_b16(oracle):
    w = wl.HCA_DECODE_1M
    inp = wl.make_inputs(w, device="cuda")
    B, N, T = w.B, w.max_blocks, w.B
    comp = torch.empty((B, N, 128), dtype=torch.bfloat16, device="cuda")
    csa.csa_compress(inp.raw_kv, inp.lens, inp.z_kv, w.m, 0, N, comp)
    torch.cuda.synchronize()
    lens = inp.lens.cpu().numpy()
    z = inp.z_kv.cpu().numpy()
    a = oracle.pool_weights(z)
    q_pos = inp.q_pos.cpu().numpy()
    qa = _bits(inp.q)
    refs = {}
    for b in (2, 11):
        L = int(lens[b])
        raw = _bits(inp.raw_kv[b:b + 1, :L])
        ck, _ = oracle.compress(raw, lens[b:b + 1], z, 0, 1 << 30)
        nb = L // w.m
        x = bf16_bits_to_f64(raw[0, :nb * w.m]).reshape(nb, w.m, 128)
        check_compress_bf16(_bits(comp[b, :nb]), ck[0, :nb], absum=np.einsum("jid,id->jd", np.abs(x), np.abs(a)), m=w.m)
        comp[b, :nb] = _to_dev(ck[0, :nb])
        refs[b] = (raw, ck)
    out = torch.empty((T, w.H, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
    ws = csa.Workspace(csa.hca_attend_workspace_size(T, w.H, N + w.W))
    csa.hca_attend(inp.q, inp.q_seq, inp.q_pos, comp, inp.raw_kv, w.m, N, w.W, 128 ** -0.5, out, lse, ws)
    ws.check()
    for b, (raw, ck) in refs.items():
        ro, rl = oracle.hca_attend(qa[b:b + 1], [0], q_pos[b:b + 1], ck, raw, w.m, w.W, 128 ** -0.5)
        check_attention(bf16_bits_to_f64(host_bits(out[b:b + 1])), lse[b:b + 1].cpu().numpy().astype(np.float64),
                        ro, rl)
    del inp, comp
    torch.cuda.empty_cache()


def test_csa_prefill_8k_sampled(oracle):
    """Chunked prefill (8192 tokens after 131072): the whole chunk runs in one
    launch configuration; 12 queries spread over the chunk are judged."""
    from long_context_sparse_03_b200.decode import CsaPrefill
    w = wl.CSA_PREFILL_8K
    inp = wl.make_inputs(w, device="cuda")
    pf = CsaPrefill(inp)
    pf.build_caches()
    i = inp
    N, T, m = w.max_blocks, w.T_new, w.m
    csa.csa_compress(i.raw_kv, i.lens, i.z_kv, m, pf.n_old, N, pf.comp)
    csa.csa_compress(i.raw_ki, i.lens, i.z_ki, m, pf.n_old, N, pf.kidx)
    torch.cuda.synchronize()
    lens = i.lens.cpu().numpy()
    raw_kv, raw_ki = _bits(i.raw_kv), _bits(i.raw_ki)
    ck, _ = oracle.compress(raw_kv, lens, i.z_kv.cpu().numpy(), 0, 1 << 30)
    kk, _ = oracle.compress(raw_ki, lens, i.z_ki.cpu().numpy(), 0, 1 << 30)
    a = oracle.pool_weights(i.z_kv.cpu().numpy())
    x = bf16_bits_to_f64(raw_kv[0, :N * m]).reshape(N, m, 128)[pf.n_old:]
    check_compress_bf16(_bits(pf.comp[0, pf.n_old:N]), ck[0, pf.n_old:N],
                        absum=np.einsum("jid,id->jd", np.abs(x), np.abs(a)), m=m)
    pf.comp[0, :N] = _to_dev(ck[0, :N])
    pf.kidx[0, :N] = _to_dev(kk[0, :N])
    # projection of all T queries on the GPU (GEMM path) vs the oracle on samples
    csa.csa_index_query(i.h, i.W_dq, i.W_uq, i.W_w, pf.q_idx, pf.w_idx, pf.ws_idx)
    sample = np.linspace(0, T - 1, 12).astype(int)
    h = _bits(i.h)[sample]
    rq, rw = oracle.index_query(h, _bits(i.W_dq), _bits(i.W_uq), _bits(i.W_w))
    gq = pf.q_idx[torch.from_numpy(sample).cuda()].cpu().numpy().astype(np.float64)
    gw = pf.w_idx[torch.from_numpy(sample).cuda()].cpu().numpy().astype(np.float64)
    for t in range(len(sample)):
        assert np.abs(gq[t] - rq[t]).max() <= 1e-5 * np.abs(rq[t]).max()
        assert np.abs(gw[t] - rw[t]).max() <= 1e-5 * np.abs(rw[t]).max()
    # selection over all T queries, the sampled ones driven by the oracle's q, w
    q32, w32 = rq.astype(np.float32), rw.astype(np.float32)
    st = torch.from_numpy(sample).cuda()
    pf.q_idx[st] = torch.from_numpy(q32).cuda()
    pf.w_idx[st] = torch.from_numpy(w32).cuda()
    csa.csa_index_select(pf.q_idx, pf.w_idx, i.q_seq, i.q_pos, pf.kidx, m, N, w.k, pf.idx, pf.idx_score, pf.ws_idx)
    pf.ws_idx.check()
    q_pos = i.q_pos.cpu().numpy()[sample]
    S = oracle.index_scores(q32.astype(np.float64), w32.astype(np.float64), np.zeros(len(sample), np.int32), q_pos,
                            kk, m, N)
    oi, _ = oracle.topk(S, q_pos, m, w.k)
    gi, gs = pf.idx[st].cpu().numpy(), pf.idx_score[st].cpu().numpy()
    kf = bf16_bits_to_f64(kk[0])
    for t in range(len(sample)):
        A = score_scale(q32[t].astype(np.float64), w32[t].astype(np.float64), kf)
        V = min((int(q_pos[t]) + 1) // m, N)
        check_topk(gi[t], gs[t], S[t], A, V, w.k)
    # attention over the oracle's selection (whole chunk in one call)
    idx_all = pf.idx.clone()
    idx_all[st] = torch.from_numpy(oi).cuda()
    csa.csa_sparse_attend(i.q, i.q_seq, i.q_pos, pf.comp, i.raw_kv, m, idx_all, w.W, 128 ** -0.5, pf.out, pf.lse,
                          pf.ws_att)
    pf.ws_att.check()
    qa = _bits(i.q)[sample]
    ro, rl = oracle.sparse_attend(qa, np.zeros(len(sample), np.int32), q_pos, ck, raw_kv, m, oi, w.W, 128 ** -0.5)
    check_attention(bf16_bits_to_f64(host_bits(pf.out[st])), pf.lse[st].cpu().numpy().astype(np.float64), ro, rl)
    del inp, pf
    torch.cuda.empty_cache()
