"""The seeded input generators (workloads/) against the recipe they state: lengths inside
their ranges, every request's slots distinct and inside the pool, unused rows poisoned,
table padding in bounds, the documented value distributions, and the same bits on every
call.  CPU only; the big pools are only drawn for the small shapes."""
import numpy as np
import pytest
import torch

import workloads as wl


@pytest.mark.parametrize("name", sorted(wl.SPECS))
def test_batch_lengths_pages_and_padding_follow_the_recipe(name):
    spec = wl.SPECS[name]
    b = wl.make_batch(spec)
    L = b.seq_lens.numpy().astype(np.int64)
    P = spec.page_size
    assert L.shape == (spec.batch,)
    if spec.mode == "extend":
        new = b.new_lens.numpy().astype(np.int64)
        prefix = L - new
        assert np.all((spec.new_lo <= new) & (new <= spec.new_hi))
        assert np.all((spec.len_lo <= prefix) & (prefix <= spec.len_hi))
        cu = b.cu_seqlens_q.numpy()
        assert cu[0] == 0 and np.array_equal(np.diff(cu), new)
    else:
        assert b.cu_seqlens_q is None
        assert np.all((spec.len_lo <= L) & (L <= spec.len_hi))
    table = b.page_table.numpy().astype(np.int64)
    num_pages = b.num_slots // P
    need = (L + P - 1) // P
    assert table.shape == (spec.batch, max(1, int(need.max())))
    # every entry (used or padding) stays inside the pool
    assert table.min() >= 0 and table.max() < num_pages
    # the pages of all requests are distinct: no two token slots alias
    used_pages = np.concatenate([table[r, :need[r]] for r in range(spec.batch)])
    assert len(np.unique(used_pages)) == len(used_pages)
    # the used-slot mask marks exactly the L_r first slots of each request's pages
    mask = b.used_slot_mask.numpy()
    assert int(mask.sum()) == int(L.sum())
    for r in range(min(spec.batch, 4)):
        slots = (table[r, :need[r], None] * P + np.arange(P)[None, :]).reshape(-1)[: L[r]]
        assert mask[slots].all()
    # spare capacity as stated
    if P == 1:
        assert b.num_slots == max(spec.pool_slots, int(L.sum()))
    else:
        assert num_pages == int(need.sum()) + int(np.ceil(need.sum() * spec.spare_pages))


@pytest.mark.parametrize("name", sorted(wl.SPECS))
def test_batches_are_the_same_bits_on_every_call(name):
    spec = wl.SPECS[name]
    a, b = wl.make_batch(spec), wl.make_batch(spec)
    assert torch.equal(a.seq_lens, b.seq_lens) and torch.equal(a.page_table, b.page_table)
    c = wl.make_batch(spec, seed=12345)
    assert not torch.equal(a.page_table, c.page_table) or not torch.equal(a.seq_lens, c.seq_lens)


def test_bf16_pools_queries_and_poisoned_rows():
    spec = wl.SPECS["decode_tiny"]
    b = wl.make_batch(spec)
    k, v = wl.make_bf16_pools(spec, b, 0)
    k2, _ = wl.make_bf16_pools(spec, b, 0)
    assert torch.equal(k.view(torch.int16), k2.view(torch.int16))
    assert k.shape == (b.num_slots, spec.hkv, spec.head_dim) and k.dtype == torch.bfloat16
    used = b.used_slot_mask
    for t in (k, v):
        assert torch.all(t.view(torch.int16)[~used] == wl.BF16_NAN)
        x = t[used].float()
        assert torch.isfinite(x).all()
        assert abs(float(x.mean())) < 0.02 and abs(float(x.std()) - 1.0) < 0.02     # N(0, 1)
    q = wl.make_bf16_queries(spec, spec.batch, 0)
    assert q.shape == (spec.batch, spec.hq, spec.head_dim)
    # a different layer draws different values
    k1, _ = wl.make_bf16_pools(spec, b, 1)
    assert not torch.equal(k[used], k1[used])


def test_peaked_rows_scale_one_percent_of_the_keys():
    spec = wl.SPECS["decode_tiny"].scaled(peaked_frac=0.01, peaked_scale=8.0, pool_slots=40000, len_lo=8000, len_hi=9000)
    b = wl.make_batch(spec)
    k, _ = wl.make_bf16_pools(spec, b, 0)
    rms = k[b.used_slot_mask].float().pow(2).mean(-1).sqrt()          # per (slot, kv head) row
    frac = float((rms > 4.0).float().mean())
    assert 0.005 < frac < 0.02


def test_fp8_pools_are_e4m3_codes_of_16_n01():
    spec = wl.SPECS["decode_fp8_llama3_8b"].scaled(batch=4, len_lo=100, len_hi=300)
    b = wl.make_batch(spec)
    k8, v8 = wl.make_fp8_pools(spec, b, 0)
    used = b.used_slot_mask
    for c in (k8, v8):
        assert c.dtype == torch.uint8
        assert torch.all(c[~used] == wl.E4M3_NAN)
        x = c[used].view(torch.float8_e4m3fn).float() * wl.FP8_SCALE
        assert torch.isfinite(x).all()
        assert float(x.abs().max()) <= 448 * wl.FP8_SCALE
        assert abs(float(x.std()) - 1.0) < 0.05                       # dequantised ~ N(0, 1)


def test_sage_layer_ranges_and_scales():
    spec = wl.SPECS["sage_decode"].scaled(batch=4, len_lo=100, len_hi=500)
    b = wl.make_batch(spec)
    lay = wl.make_sage_layer(spec, b, 0)
    used = b.used_slot_mask
    assert lay.q8.dtype == torch.int8 and int(lay.q8.min()) >= -127 and int(lay.q8.max()) <= 127
    assert int(lay.k8[used].min()) >= -127
    assert torch.all(lay.v8[~used] == wl.E4M3_NAN)
    v = lay.v8[used].view(torch.float8_e4m3fn).float()
    assert torch.isfinite(v).all() and abs(float(v.std()) - 16.0) < 1.0
    for sf in (lay.sf_q, lay.sf_k, lay.sf_v):
        ln = torch.log(sf)
        assert torch.all(sf > 0) and abs(float(ln.mean()) + 4.0) < 0.2 and abs(float(ln.std()) - 0.5) < 0.1
    assert lay.sf_k.shape == (b.num_slots // 64, spec.hkv)
    assert abs(float(lay.v_mean.std()) - 0.1) < 0.02


def test_block_mask_density():
    spec = wl.SPECS["sage_sparse_decode"]
    b = wl.make_batch(spec)
    m = wl.make_block_mask(spec, b)
    assert m.shape == b.page_table.shape and m.dtype == torch.uint8
    assert set(np.unique(m.numpy())) <= {0, 1}
    assert abs(float(m.float().mean()) - spec.density) < 0.01


def test_decode_kv_bytes_closed_form():
    # two requests of 3 and 70 keys, page size 64: K+V 73 keys x Hkv 2 x D 128 x 2 B x 2, 1 + 2 pages
    # of table entries, Q and O of 2 requests x 4 heads x 128 x 2 B each
    got = wl.decode_kv_bytes([3, 70], 2, 128, 2, 64, 4, 2, 2)
    assert got == 73 * 2 * 128 * 2 * 2 + 3 * 4 + 2 * 4 * 128 * 4
