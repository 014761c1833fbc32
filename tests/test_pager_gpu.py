"""Continuous batching on the GPU with the host pager (include/gqa_pager.h): sequences
join with a prompt, take decode steps through gqa_decode_step with the block table,
positions and lengths the pager hands out, finish and give their pages back, and later
sequences reuse those pages (whose stale rows are poisoned with NaN in between).  Every
step's output is checked against the oracle over a host copy of the pools kept in step
with the oracle's kv_append."""
import numpy as np
import pytest
import torch

import gqa_decode_attention_04_b200 as gq
import oracle
from parity import assert_close, gpu_f64
from workloads import bf16_bits

pytestmark = pytest.mark.gpu


def _bf16_from_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("H,Hk,D,ps", [(8, 2, 128, 16), (96, 1, 128, 64), (4, 1, 64, 16)])
def test_continuous_batching_with_the_pager(cuda_device, H, Hk, D, ps):
    rng = np.random.default_rng(11 + H)
    gen = torch.Generator().manual_seed(11 + H)
    P, S, MB = 48, 6, 12
    pager = gq.Pager(P, ps, S, MB)
    nan_bits = np.uint16(0x7FC0)
    k_host = np.full((P, Hk, ps, D), nan_bits, dtype=np.uint16)   # oracle's copy of the pools
    v_host = np.full((P, Hk, ps, D), nan_bits, dtype=np.uint16)
    k_dev = _bf16_from_bits(k_host).to(cuda_device)
    v_dev = _bf16_from_bits(v_host).to(cuda_device)
    scale = D ** -0.5
    active = []
    steps_checked = 0
    for step in range(12):
        # finish some sequences: their pages go back (and are poisoned, as a stale cache)
        for s in list(active):
            if rng.random() < 0.2:
                bt_row, _ = pager.gather([s])
                pages = [p for p in bt_row[0].tolist() if p >= 0]
                pager.release(s)
                active.remove(s)
                k_host[pages] = nan_bits
                v_host[pages] = nan_bits
                k_dev[pages] = float("nan")
                v_dev[pages] = float("nan")
        # admit new sequences with a prompt while slots and pages allow
        for s in range(S):
            if s in active or rng.random() < 0.4:
                continue
            n = int(rng.integers(1, 5 * ps))
            try:
                pager.extend(s, n)
            except gq.GQAError as e:
                assert e.status == -6
                continue
            bt_row, _ = pager.gather([s])
            t = np.arange(n)
            pages, rows = bt_row[0].numpy()[t // ps], t % ps
            kp = bf16_bits(torch.randn(n, Hk, D, generator=gen).to(torch.bfloat16))
            vp = bf16_bits(torch.randn(n, Hk, D, generator=gen).to(torch.bfloat16))
            k_host[pages, :, rows, :] = kp
            v_host[pages, :, rows, :] = vp
            pi, ri = torch.from_numpy(pages).long().to(cuda_device), torch.from_numpy(rows).long().to(cuda_device)
            k_dev[pi, :, ri, :] = _bf16_from_bits(kp).to(cuda_device)
            v_dev[pi, :, ri, :] = _bf16_from_bits(vp).to(cuda_device)
            active.append(s)
        if not active:
            continue
        batch = list(active)
        rng.shuffle(batch)            # batch order is the caller's, not the slots'
        try:
            pos, lens = pager.step(batch)
        except gq.GQAError as e:
            assert e.status == -6
            continue
        bt, lens2 = pager.gather(batch)
        assert torch.equal(lens, lens2)
        B = len(batch)
        q = torch.randn(B, H, D, generator=gen).to(torch.bfloat16)
        kn = torch.randn(B, Hk, D, generator=gen).to(torch.bfloat16)
        vn = torch.randn(B, Hk, D, generator=gen).to(torch.bfloat16)
        out = gq.decode_step(q.to(cuda_device), kn.to(cuda_device), vn.to(cuda_device), k_dev, v_dev,
                             bt.to(cuda_device), pos.to(cuda_device), lens.to(cuda_device), scale=scale)
        gq.check_device_error()
        k_host, v_host = oracle.kv_append(k_host, v_host, bf16_bits(kn), bf16_bits(vn), bt.numpy(), pos.numpy())
        assert np.array_equal(bf16_bits(k_dev), k_host) and np.array_equal(bf16_bits(v_dev), v_host)
        want = oracle.paged_decode_attention(bf16_bits(q), k_host, v_host, bt.numpy(), lens.numpy(), scale)
        assert_close(gpu_f64(out), want, what=f"step {step}, batch {batch}")
        steps_checked += 1
    assert steps_checked >= 6
    # every page is back once every sequence finishes
    for s in active:
        pager.release(s)
    assert pager.free_pages == P


@pytest.mark.parametrize("H,Hk,Q", [(8, 2, 4), (32, 2, 4), (4, 1, 8)])
def test_speculative_steps_with_the_pager(cuda_device, H, Hk, Q):
    """Draft-and-verify: each step every sequence takes q_len draft tokens (pager.extend;
    gqa_multi_query_step appends their K/V and attends with per-token windows), then keeps
    a random number of them (pager.truncate).  Rejected rows are poisoned with NaN, as a
    stale cache would be, and must never be read again."""
    D, ps, S, MB, P = 128, 16, 4, 16, 40
    rng = np.random.default_rng(31 + H + Q)
    gen = torch.Generator().manual_seed(32 + H + Q)
    pager = gq.Pager(P, ps, S, MB)
    nan = np.uint16(0x7FC0)
    k_host = np.full((P, Hk, ps, D), nan, dtype=np.uint16)
    v_host = np.full((P, Hk, ps, D), nan, dtype=np.uint16)
    k_dev = _bf16_from_bits(k_host).to(cuda_device)
    v_dev = _bf16_from_bits(v_host).to(cuda_device)
    scale = D ** -0.5
    seqs = list(range(S))
    for s in seqs:  # prompts
        n = int(rng.integers(1, 60))
        pager.extend(s, n)
        bt_row, _ = pager.gather([s])
        t = np.arange(n)
        pages, rows = bt_row[0].numpy()[t // ps], t % ps
        kp = bf16_bits(torch.randn(n, Hk, D, generator=gen).to(torch.bfloat16))
        vp = bf16_bits(torch.randn(n, Hk, D, generator=gen).to(torch.bfloat16))
        k_host[pages, :, rows, :] = kp
        v_host[pages, :, rows, :] = vp
        pi = torch.from_numpy(pages).long().to(cuda_device)
        ri = torch.from_numpy(rows).long().to(cuda_device)
        k_dev[pi, :, ri, :] = _bf16_from_bits(kp).to(cuda_device)
        v_dev[pi, :, ri, :] = _bf16_from_bits(vp).to(cuda_device)
    for step in range(6):
        _, before = pager.gather(seqs)
        for s in seqs:
            pager.extend(s, Q)
        bt, lens = pager.gather(seqs)
        pos = before.clone()
        B = len(seqs)
        q = torch.randn(B, Q, H, D, generator=gen).to(torch.bfloat16)
        kn = torch.randn(B, Q, Hk, D, generator=gen).to(torch.bfloat16)
        vn = torch.randn(B, Q, Hk, D, generator=gen).to(torch.bfloat16)
        out = gq.multi_query_step(q.to(cuda_device), kn.to(cuda_device), vn.to(cuda_device), k_dev, v_dev,
                                  bt.to(cuda_device), pos.to(cuda_device), lens.to(cuda_device), scale=scale)
        gq.check_device_error()
        k_host, v_host = oracle.kv_append_multi(k_host, v_host, bf16_bits(kn), bf16_bits(vn), bt.numpy(),
                                                pos.numpy())
        assert np.array_equal(bf16_bits(k_dev), k_host) and np.array_equal(bf16_bits(v_dev), v_host)
        want = oracle.paged_multi_query_attention(bf16_bits(q), k_host, v_host, bt.numpy(), lens.numpy(), scale)
        assert_close(gpu_f64(out), want, what=f"step {step}")
        # verification: keep a random prefix of each sequence's drafts
        for b, s in enumerate(seqs):
            keep = int(rng.integers(0, Q + 1))
            new_len = int(before[b]) + keep
            row = bt[b].numpy()
            for t in range(new_len, int(lens[b])):  # rejected rows: stale from now on
                pg, sl = int(row[t // ps]), t % ps
                k_host[pg, :, sl, :] = nan
                v_host[pg, :, sl, :] = nan
                k_dev[pg, :, sl, :] = float("nan")
                v_dev[pg, :, sl, :] = float("nan")
            pager.truncate(s, new_len)
    assert pager.free_pages + sum(-(-pager.seq_len(s) // ps) for s in seqs) == P
