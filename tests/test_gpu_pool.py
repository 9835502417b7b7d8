"""GPU parity of the paged pool (ragged batching): sequences of different lengths in
one buffer, decoded together by duo_pool_decode_step, against the fp64 oracle per
(layer, sequence); cached rows read back bit for bit through the block table."""
import numpy as np
import pytest
import torch

import oracle
from head_split_kv_duo_b200 import duo, inputs
from head_split_kv_duo_b200.duo import DuoPool
from parity import assert_close, bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _history(nseq, layers, T, Hkv, seed):
    k = inputs.randn((nseq, layers, T, Hkv, 128), seed, device=DEV)
    v = inputs.randn((nseq, layers, T, Hkv, 128), seed + 1, device=DEV)
    return k, v


def _check_rows(pool, seq, layer, k, v, length):
    """Retrieval rows through the block table and ring slots, bit for bit; the rows of
    the sequence's last page past its length and its unwritten ring slots are zero."""
    Hkv, S, W = pool.kv_heads, pool.S, pool.W
    mask = pool.mask[layer].tolist()
    ridx = [g for g in range(Hkv) if mask[g]]
    sidx = [g for g in range(Hkv) if not mask[g]]
    rk = pool.region(layer, duo.DUO_REGION_RETR_K).view(torch.int16).view(pool.num_pages, len(ridx), 128, 128)
    rv = pool.region(layer, duo.DUO_REGION_RETR_V).view(torch.int16).view(pool.num_pages, len(ridx), 128, 128)
    kb, vb = k.view(torch.int16), v.view(torch.int16)
    for lp in range((length + 127) // 128):
        page = pool.page(seq, lp)
        rows = min(128, length - lp * 128)
        for i, g in enumerate(ridx):
            assert torch.equal(rk[page, i, :rows], kb[lp * 128:lp * 128 + rows, g])
            assert torch.equal(rv[page, i, :rows], vb[lp * 128:lp * 128 + rows, g])
            assert not rk[page, i, rows:].any() and not rv[page, i, rows:].any()
    if sidx:
        sk = pool.region(layer, duo.DUO_REGION_STRM_K).view(torch.int16).view(pool.max_seqs, len(sidx), S + W, 128)
        sv = pool.region(layer, duo.DUO_REGION_STRM_V).view(torch.int16).view(pool.max_seqs, len(sidx), S + W, 128)
        replay = oracle.ring_replay(S, W, [length])[0] if length > 0 else -np.ones(S + W, dtype=np.int64)
        for i, g in enumerate(sidx):
            for slot in range(S + W):
                pos = int(replay[slot])
                if pos >= 0:
                    assert torch.equal(sk[seq, i, slot], kb[pos, g]) and torch.equal(sv[seq, i, slot], vb[pos, g])
                else:
                    assert not sk[seq, i, slot].any() and not sv[seq, i, slot].any()


def _run_and_check(Hq, Hkv, layers, S, W, prompts, steps, num_pages, seed, layers_per_call, check_rows=True):
    G = Hq // Hkv
    mask = inputs.retrieval_mask(layers, Hkv, Hkv // 2, seed=seed)
    T = max(prompts) + steps
    pool = DuoPool(layers, Hkv, mask, S, W, max_seqs=len(prompts) + 2, max_len=T + 4, num_pages=num_pages, q_heads=Hq)
    seqs = [pool.open() for _ in prompts]
    K, V = _history(len(prompts), layers, T, Hkv, seed)
    Q = inputs.randn((steps, layers, len(prompts), Hq, 128), seed + 2, device=DEV)
    for i, s in enumerate(seqs):
        for l in range(layers):
            if prompts[i] > 0:
                pool.append_kv(l, s, K[i, l, :prompts[i]].contiguous(), V[i, l, :prompts[i]].contiguous())
    outs, lses = [], []
    for t in range(steps):
        pos = torch.tensor([prompts[i] + t for i in range(len(prompts))], device=DEV)
        k = torch.stack([K[torch.arange(len(prompts)), l, pos] for l in range(layers)])  # [layers][nseq][Hkv][d]
        v = torch.stack([V[torch.arange(len(prompts)), l, pos] for l in range(layers)])
        o = torch.empty(layers, len(prompts), Hq, 128, dtype=torch.bfloat16, device=DEV)
        lse = torch.empty(layers, len(prompts), Hq, dtype=torch.float32, device=DEV)
        for l0 in range(0, layers, layers_per_call):
            sl = slice(l0, l0 + layers_per_call)
            pool.decode_step(l0, layers_per_call, seqs, Q[t, sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(),
                             out=o[sl], lse=lse[sl])
        outs.append(o)
        lses.append(lse)
    torch.cuda.synchronize()
    assert pool.device_status() == 0
    for i, s in enumerate(seqs):
        for l in range(layers):
            assert pool.len(s, l) == prompts[i] + steps
            if check_rows:
                _check_rows(pool, s, l, K[i, l, :prompts[i] + steps], V[i, l, :prompts[i] + steps], prompts[i] + steps)
    got = torch.stack(outs).float().cpu().numpy()          # [steps][layers][nseq][Hq][d]
    got_lse = torch.stack(lses).cpu().numpy()
    for i in range(len(prompts)):
        for l in range(layers):
            want, want_lse = [], []
            for t in range(steps):
                p = prompts[i] + t
                w, wl = oracle.attend(bits(Q[t, l, i][None, None]), bits(K[i, l, :p + 1][None]),
                                      bits(V[i, l, :p + 1][None]), mask[l].numpy().astype(bool), S, W, pos0=p)
                want.append(w[0, 0])
                want_lse.append(wl[0, 0])
            assert_close(got[:, l, i], np.stack(want), torch.bfloat16, got_lse[:, l, i], np.stack(want_lse),
                         f"pool seq {i} (prompt {prompts[i]}) layer {l}")
    return pool, seqs


@pytest.mark.parametrize("layers_per_call", [1, 3])
def test_pool_ragged_decode_small(layers_per_call):
    """GQA 16 q / 4 kv heads, 3 layers, S 4, W 40: prompts of 0, 1, 17, 127, 128, 300 and
    700 tokens (first token, around a page boundary, ring wrapping), 3 steps."""
    _run_and_check(16, 4, 3, 4, 40, [0, 1, 17, 127, 128, 300, 700], 3, 64, 50, layers_per_call)


def test_pool_ragged_decode_llama3_shape():
    """Llama-3-8B GQA layer shape (32 q / 8 kv heads, 4 retrieval, S 16, W 512), 8
    sequences from 64 to 32K tokens in one step, 2 steps, both layers in one launch."""
    prompts = [1000, 5000, 12000, 32768, 300, 64, 2048, 20000]
    _run_and_check(32, 8, 2, 16, 512, prompts, 2, sum((p + 130) // 128 + 1 for p in prompts), 60, 2,
                   check_rows=False)


def test_pool_recycled_sequences():
    """Closing sequences returns their pages and slots; sequences opened in them start
    from clean rows and decode like fresh ones."""
    Hq, Hkv, layers, S, W = 8, 4, 2, 2, 24
    pool, seqs = _run_and_check(Hq, Hkv, layers, S, W, [200, 50, 129], 2, 12, 70, 2)
    free = pool.free_pages()
    pool.close_seq(seqs[0])
    pool.close_seq(seqs[2])
    assert pool.free_pages() == free + 2 + 2
    mask = pool.mask
    new = [pool.open(), pool.open()]
    assert sorted(new) == sorted([seqs[0], seqs[2]])
    K, V = _history(2, layers, 40, Hkv, 71)
    Q = inputs.randn((layers, 2, Hq, 128), 73, device=DEV)
    for i, s in enumerate(new):
        for l in range(layers):
            pool.append_kv(l, s, K[i, l, :30].contiguous(), V[i, l, :30].contiguous())
    k = K[:, :, 30].transpose(0, 1).contiguous()
    v = V[:, :, 30].transpose(0, 1).contiguous()
    o, lse = pool.decode_step(0, layers, new, Q, k, v)
    torch.cuda.synchronize()
    for i, s in enumerate(new):
        for l in range(layers):
            _check_rows(pool, s, l, K[i, l, :31], V[i, l, :31], 31)
            w, wl = oracle.attend(bits(Q[l, i][None, None]), bits(K[i, l, :31][None]), bits(V[i, l, :31][None]),
                                  mask[l].numpy().astype(bool), S, W, pos0=30)
            assert_close(o[l, i].float().cpu().numpy()[None], w[0], torch.bfloat16, lse[l, i].cpu().numpy()[None],
                         wl[0], f"recycled seq {i} layer {l}")
