"""Input-generator checks: shapes against the pages' printed numbers, determinism."""
import os

import torch

import wan_inputs as wi

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "wan_token_grids.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line.split())
    return rows


def test_token_grid_matches_pages():
    for row in _golden():
        if row[0] == "grid":
            w, h, fr, F, H, W, S = map(int, row[1:])
            assert wi.dit_token_grid(w, h, fr) == (F, H, W)
            assert F * H * W == S


def test_a14b_attention_shape_matches_pages():
    for row in _golden():
        if row[0] == "attn":
            S, heads, hd, hidden = map(int, row[1:])
            w = wi.BY_NAME["a14b_720p_81f_b1"]
            assert (w.seq_len, w.heads, wi.HEAD_DIM, w.dim) == (S, heads, hd, hidden)
            assert wi.dit_token_grid(1280, 720, 81) == w.grid


def test_bench_workload_is_480p_81f_cfg():
    w = wi.BENCH_WORKLOAD
    assert w.grid == (21, 30, 52) and w.batch == 2 and w.heads == 40


def test_generators_are_seeded():
    a = wi.packed_qkv(1, 10, 2, seed=5)
    b = wi.packed_qkv(1, 10, 2, seed=5)
    c = wi.packed_qkv(1, 10, 2, seed=6)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))
    gq, gk = wi.gammas(3)
    assert gq.shape == (384,) and float(gq.float().min()) >= 0.5 and float(gq.float().max()) <= 1.5
    assert not torch.equal(gq, gk)


def test_sample_rows_cover_tails():
    r = wi.sample_rows(32760, 64, seed=0).tolist()
    assert r[0] == 0 and r[-1] == 32759
    assert set(range(32640, 32760)) <= set(r)
