"""GPU parity of the decode step (axis_attn_decode) against the oracle.

The oracle reads a contiguous cache [B, Smax, Hkv, D]; the test scatters the
same rows into a shuffled pool of pages, fills the block table (entries past a
sequence's last page hold -1, which the kernel must never touch) and compares
O and LSE with the tolerances of the other tests (O max abs <= 1e-2, LSE max
abs <= 1e-4).  Cases cover both head dims, GQA groups 1..8 (including 3),
page sizes 8..256, ragged lengths (1, around page and piece edges), batches
that take the split-K path and batches that do not, both kernel
configurations (deep for few items, wide for many), and bad device-side
indices, which must be reported as AXIS_ATTN_ERR_INDEX without an access.
Every case runs on both pool layouts: [num_pages, page_size, Hkv, D]
(axis_attn_decode) and the head-major [num_pages, Hkv, page_size, D]
(axis_attn_decode_hnd), the latter a transposed copy of the same pool.
"""
import math

import numpy as np
import pytest
import torch

import causal_attention_fwd_b200 as aa

pytestmark = pytest.mark.gpu

TOL_O, TOL_LSE = 1e-2, 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_fwd_b200 import build

    build.build()


def paged(k, v, lens, page_size, seed, extra_pages=3):
    """Scatter contiguous caches [B, Smax, Hkv, D] into a shuffled page pool."""
    B, Smax, Hkv, D = k.shape
    max_pages = (Smax + page_size - 1) // page_size
    need = [(int(L) + page_size - 1) // page_size for L in lens]
    num_pages = sum(need) + extra_pages
    order = np.random.default_rng(seed).permutation(num_pages)
    kc = torch.zeros((num_pages, page_size, Hkv, D), dtype=k.dtype)
    vc = torch.zeros_like(kc)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    n = 0
    for b in range(B):
        for p in range(need[b]):
            page = int(order[n])
            n += 1
            table[b, p] = page
            rows = slice(p * page_size, min((p + 1) * page_size, int(lens[b])))
            cnt = rows.stop - rows.start
            kc[page, :cnt] = k[b, rows]
            vc[page, :cnt] = v[b, rows]
    return kc, vc, table, num_pages


def as_layout(kc, vc, layout):
    """The pool in the requested layout ("HND" swaps the page-row and head axes)."""
    if layout == "HND":
        return kc.transpose(1, 2).contiguous(), vc.transpose(1, 2).contiguous()
    return kc, vc


def run_case(oracle_mod, B, Hq, Hkv, D, Smax, page_size, lens, seed, layout="NHD"):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    lens = np.asarray(lens, np.int32)
    sc = 1.0 / math.sqrt(D)
    kc, vc, table, num_pages = paged(k, v, lens, page_size, seed)
    kc, vc = as_layout(kc, vc, layout)
    dev = torch.device("cuda:0")
    o, lse = aa.attention_decode(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev),
                                 torch.from_numpy(lens).to(dev), scale=sc, layout=layout)
    aa.check_status()
    ro, rl = oracle_mod.attn_decode(q, k, v, lens, sc)
    eo = float((o.cpu().double() - torch.from_numpy(ro)).abs().max())
    el = float((lse.cpu().double() - torch.from_numpy(rl)).abs().max())
    return eo, el


CASES = [
    # B, Hq, Hkv, D, Smax, page_size, lens
    (1, 1, 1, 64, 1, 8, [1]),
    (3, 4, 4, 64, 100, 16, [1, 31, 100]),
    (2, 12, 4, 64, 1024, 16, [1024, 517]),           # the axiomlm model's heads and block size
    (4, 8, 1, 128, 300, 32, [32, 33, 64, 299]),
    (2, 6, 2, 128, 700, 64, [700, 65]),
    (5, 16, 2, 64, 257, 256, [256, 257, 1, 128, 200]),
    (1, 32, 8, 128, 8192, 64, [8192]),               # one long sequence: split-K
    (2, 24, 8, 64, 5000, 8, [4999, 3]),               # G = 3, small pages, split-K
    (64, 32, 8, 128, 600, 16, list(range(9, 9 + 64 * 9, 9))),  # many sequences: no split
    # more than 32 pieces of 32 keys per CTA: the producer reads the block
    # table in several blocks of 32 pieces (3 at 2100 keys, 2 at 1500)
    (40, 8, 8, 64, 2100, 8, [2100, 1, 1024, 1025, 2047, 2048, 2049, 33] * 5),
    (40, 16, 8, 128, 1500, 16, [1500, 1023, 1056, 17, 1499] * 8),
    # more items than the wide D = 64 configuration's resident CTAs (800 > 740):
    # the wide kernel, some CTAs walking two items (the cases above with at most
    # 444 items at D = 64 / 296 at D = 128 run the deep configuration)
    (200, 8, 4, 64, 300, 16, [300, 1, 17, 256, 299] * 40),
    # 128 splits of 256 keys (more than the merge kernel's 32 splits per pass of
    # its warps), the last 10 past the end of the sequence (weight 0)
    (1, 4, 2, 64, 32768, 16, [30001]),
]


@pytest.mark.parametrize("layout", ["NHD", "HND"])
@pytest.mark.parametrize("B,Hq,Hkv,D,Smax,ps,lens", CASES)
def test_decode_matches_oracle(oracle_mod, B, Hq, Hkv, D, Smax, ps, lens, layout):
    eo, el = run_case(oracle_mod, B, Hq, Hkv, D, Smax, ps, lens, seed=3000 + B + Hq + D + Smax + ps, layout=layout)
    print(f"{layout} B{B} Hq{Hq} Hkv{Hkv} D{D} S{Smax} ps{ps}: O {eo:.2e} LSE {el:.2e}")
    assert eo <= TOL_O and el <= TOL_LSE


def test_decode_workspace_is_split_dependent():
    # one sequence of 8192 keys over 8 kv heads is split; 64 x 8 units are not
    assert aa.axis_attn_decode_workspace_bytes(1, 32, 8, 128, 64, 128) > 0
    assert aa.axis_attn_decode_workspace_bytes(64, 32, 8, 128, 16, 38) == 0
    assert aa.axis_attn_decode_workspace_bytes(1, 32, 8, 96, 64, 128) == 0  # unsupported D


@pytest.mark.parametrize("layout", ["NHD", "HND"])
def test_decode_bad_indices_are_reported_not_used(oracle_mod, layout):
    B, Hq, Hkv, D, Smax, ps = 2, 4, 2, 64, 64, 16
    g = torch.Generator().manual_seed(9)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    lens = np.array([64, 40], np.int32)
    kc, vc, table, num_pages = paged(k, v, lens, ps, 9)
    kc, vc = as_layout(kc, vc, layout)
    dev = torch.device("cuda:0")
    args = [t.to(dev) for t in (q, kc, vc)]
    bad = table.clone()
    bad[1, 1] = num_pages + 1000  # inside sequence 1's length
    aa.attention_decode(*args, bad.to(dev), torch.from_numpy(lens).to(dev), scale=D ** -0.5, layout=layout)
    assert aa.axis_attn_get_status(aa.binding._stream(None)) == 8  # AXIS_ATTN_ERR_INDEX
    bad_len = torch.tensor([64, 10 ** 6], dtype=torch.int32)
    aa.attention_decode(*args, table.to(dev), bad_len.to(dev), scale=D ** -0.5, layout=layout)
    assert aa.axis_attn_get_status(aa.binding._stream(None)) == 8
    # the same call with good indices is exact afterwards
    o, lse = aa.attention_decode(*args, table.to(dev), torch.from_numpy(lens).to(dev), scale=D ** -0.5,
                                 layout=layout)
    aa.check_status()
    ro, rl = oracle_mod.attn_decode(q, k, v, lens, D ** -0.5)
    assert float((o.cpu().double() - torch.from_numpy(ro)).abs().max()) <= TOL_O


# ---- several new tokens per sequence (axis_attn_decode_q)

def run_case_q(oracle_mod, B, q_len, Hq, Hkv, D, Smax, page_size, lens, seed, layout="NHD"):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, q_len, Hq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    lens = np.asarray(lens, np.int32)
    sc = 1.0 / math.sqrt(D)
    kc, vc, table, num_pages = paged(k, v, lens, page_size, seed)
    kc, vc = as_layout(kc, vc, layout)
    dev = torch.device("cuda:0")
    o, lse = aa.attention_decode(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev),
                                 torch.from_numpy(lens).to(dev), scale=sc, layout=layout)
    aa.check_status()
    assert o.shape == (B, q_len, Hq, D) and lse.shape == (B, Hq, q_len)
    ro, rl = oracle_mod.attn_decode_q(q, k, v, lens, sc)
    eo = float((o.cpu().double() - torch.from_numpy(ro)).abs().max())
    el = float((lse.cpu().double() - torch.from_numpy(rl)).abs().max())
    return eo, el


CASES_Q = [
    # B, q_len, Hq, Hkv, D, Smax, page_size, lens
    (2, 2, 8, 8, 64, 100, 16, [2, 100]),               # G = 1: 2 of a tile's 16 rows
    (3, 4, 12, 4, 64, 300, 16, [4, 33, 300]),          # G = 3: 12 rows; len = q_len
    (2, 3, 32, 4, 128, 700, 64, [700, 35]),            # G = 8: 24 rows -> 2 tiles, the second ragged
    (1, 16, 2, 2, 64, 8192, 32, [8190]),               # one long sequence: split-K, 16 new tokens
    (1, 5, 24, 8, 64, 5000, 8, [4999]),                # G = 3, q_len 5: tiles ragged; split-K
    (48, 2, 16, 8, 128, 600, 16, [600, 2, 37, 599] * 12),  # many sequences, no split
    (40, 8, 8, 8, 64, 2100, 8, [2100, 8, 1024, 1025, 2047, 2048, 2049, 33] * 5),
    # a split boundary (8192) among the new tokens: the first 8 of them see no
    # key of the last split, whose partial result must weigh nothing
    (1, 16, 2, 2, 64, 8320, 32, [8200]),
    (2, 8, 32, 4, 64, 500, 16, [500, 9]),              # G = 8: 64 rows -> 4 tiles of 16
    # 16-row tiles with more items than the deep configuration takes in one wave
    # (the wide kernel): 320 items at D = 64, 384 at D = 128
    (80, 4, 16, 4, 64, 200, 16, [200, 4, 63, 150] * 20),
    (48, 8, 16, 8, 128, 300, 32, [300, 8, 100, 257] * 12),
]


@pytest.mark.parametrize("layout", ["NHD", "HND"])
@pytest.mark.parametrize("B,q_len,Hq,Hkv,D,Smax,ps,lens", CASES_Q)
def test_decode_q_matches_oracle(oracle_mod, B, q_len, Hq, Hkv, D, Smax, ps, lens, layout):
    eo, el = run_case_q(oracle_mod, B, q_len, Hq, Hkv, D, Smax, ps, lens,
                        seed=7000 + B + q_len + Hq + D + Smax + ps, layout=layout)
    print(f"{layout} B{B} q{q_len} Hq{Hq} Hkv{Hkv} D{D} S{Smax} ps{ps}: O {eo:.2e} LSE {el:.2e}")
    assert eo <= TOL_O and el <= TOL_LSE


def test_decode_q_one_token_is_the_decode_step():
    B, Hq, Hkv, D, Smax, ps = 4, 8, 2, 64, 300, 16
    g = torch.Generator().manual_seed(71)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    lens = np.array([300, 1, 17, 256], np.int32)
    kc, vc, table, _ = paged(k, v, lens, ps, 71)
    dev = torch.device("cuda:0")
    args = [t.to(dev) for t in (kc, vc, table)] + [torch.from_numpy(lens).to(dev)]
    o1, l1 = aa.attention_decode(q.to(dev), *args, scale=0.125)
    oq, lq = aa.attention_decode(q.to(dev)[:, None], *args, scale=0.125)
    aa.check_status()
    assert torch.equal(o1, oq[:, 0]) and torch.equal(l1, lq[:, :, 0])


def test_decode_q_short_length_is_reported(oracle_mod):
    B, q_len, Hq, Hkv, D, Smax, ps = 2, 4, 4, 2, 64, 64, 16
    g = torch.Generator().manual_seed(72)
    q = torch.randn((B, q_len, Hq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Smax, Hkv, D), generator=g).to(torch.bfloat16)
    lens = np.array([64, 40], np.int32)
    kc, vc, table, _ = paged(k, v, lens, ps, 72)
    dev = torch.device("cuda:0")
    args = [t.to(dev) for t in (q, kc, vc, table)]
    aa.attention_decode(*args, torch.tensor([64, 3], dtype=torch.int32, device=dev), scale=0.125)
    assert aa.axis_attn_get_status(aa.binding._stream(None)) == 8  # a sequence shorter than its new tokens
    # the same call with good lengths is exact afterwards
    o, lse = aa.attention_decode(*args, torch.from_numpy(lens).to(dev), scale=0.125)
    aa.check_status()
    ro, rl = oracle_mod.attn_decode_q(q, k, v, lens, 0.125)
    assert float((o.cpu().double() - torch.from_numpy(ro)).abs().max()) <= TOL_O
    assert float((lse.cpu().double() - torch.from_numpy(rl)).abs().max()) <= TOL_LSE
