"""Pins of the float64 oracle against things other than itself.

Each test fixes the oracle to a fact from the pages or from mathematics:
  - brute force: PyTorch's float64 CPU scaled_dot_product_attention with an
    explicit boolean mask (on fixed cases and on 24 seeded random shapes,
    windows and dtypes), and an independent pure-Python loop;
  - window = context (or more) equals unlimited, and window 0 is full causal
    (gllm PR #116 "feat(backend): sliding-window PagedAttention",
    "Verification": "Window = context matches unlimited");
  - closed forms: window 1 returns v_p exactly, equal keys give the mean of
    the visible values, two visible tokens give logistic weights;
  - invariants: physical block placement does not matter (that page's
    "scattered out-of-order blocks"), any split-K partition count gives the
    same result (ExecuTorch PR #18759, split-K merge), softmax weights sum to
    one and vanish outside the visible range;
  - the hand-derived visible ranges in tests/golden/visible_ranges.txt;
  - FP8 e4m3 caches: every one of the 256 codes decodes to the value torch's
    float8_e4m3fn conversion gives, a handful of codes to their closed forms
    (OCP 8-bit floating point formats: bias 7, no infinities, 448 largest),
    and attention over FP8 codes equals float64 SDPA over the dequantised
    caches, with k_scale acting on the logits and v_scale on the output.
A plausible slip in the oracle (a dropped scale, an off-by-one window edge, a
wrong GQA head map, a swapped K/V, a bad block lookup) fails at least one.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_474_b200.workloads import bf16_bits, config_workload, make_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "visible_ranges.txt")


def problem_of(w, window=None, windows="keep"):
    ws = w.windows if windows == "keep" else windows
    return oracle.Problem(
        bf16_bits(w.q), bf16_bits(w.k_cache), bf16_bits(w.v_cache),
        w.block_tables.numpy(), w.seq_lens.numpy(), w.query_lens.numpy(),
        w.scale, w.window if window is None else window,
        None if ws is None else np.asarray(ws, dtype=np.int32),
        k_scale=w.k_scale, v_scale=w.v_scale, q_scale=w.q_scale)


def cache_values(c, s):
    """float64 values of a cache: bf16 as is, FP8 codes decoded by torch's own
    float8_e4m3fn conversion and multiplied by their per-tensor scale."""
    if c.dtype == torch.uint8:
        return c.view(torch.float8_e4m3fn).double() * s
    return c.double()


def dense_kv(w, b):
    """K and V of row b gathered into [S, Hkv, D] float64 by walking its block
    table (written here independently of the oracle)."""
    S = int(w.seq_lens[b])
    bs = w.block_size
    kc = cache_values(w.k_cache, w.k_scale)
    vc = cache_values(w.v_cache, w.v_scale)
    ks, vs = [], []
    for t in range(S):
        phys = int(w.block_tables[b, t // bs])
        ks.append(kc[phys, :, t % bs, :])
        vs.append(vc[phys, :, t % bs, :])
    return torch.stack(ks), torch.stack(vs)


def sdpa_reference(w, window_of_row):
    """All outputs via torch float64 SDPA with an explicit boolean mask."""
    outs = []
    qoff = 0
    G = w.num_q_heads // w.num_kv_heads
    for b in range(w.batch):
        S, L = int(w.seq_lens[b]), int(w.query_lens[b])
        if L == 0:
            continue
        k, v = dense_kv(w, b)                      # [S, Hkv, D]
        k = k.permute(1, 0, 2).repeat_interleave(G, dim=0)  # [Hq, S, D]
        v = v.permute(1, 0, 2).repeat_interleave(G, dim=0)
        q = cache_values(w.q[qoff:qoff + L], w.q_scale).permute(1, 0, 2)  # [Hq, L, D]
        pos = torch.arange(S - L, S).unsqueeze(1)
        t = torch.arange(S).unsqueeze(0)
        win = window_of_row(b)
        mask = t <= pos
        if win > 0:
            mask &= t > pos - win
        o = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, attn_mask=mask, scale=w.scale)
        outs.append(o.permute(1, 0, 2))
        qoff += L
    return torch.cat(outs).numpy()


def small_mixed(seed=11, bs=4, window=0, windows=None, d=16):
    """GQA group 3, mixed query lengths (decode, MTP, prefill chunk)."""
    return make_workload(seq_lens=[9, 23, 5, 31], query_lens=[1, 3, 5, 2],
                         num_q_heads=6, num_kv_heads=2, head_dim=d,
                         block_size=bs, window=window, windows=windows,
                         dist="normal", seed=seed, scale=0.3)


@pytest.mark.parametrize("window", [0, 8])
def test_tiny_workload_matches_torch_sdpa(window):
    w = config_workload(1, window=window)
    got = oracle.decode(problem_of(w))
    ref = sdpa_reference(w, lambda b: window)
    assert np.max(np.abs(got - ref)) <= 1e-12


@pytest.mark.parametrize("window,windows", [(0, None), (2, None), (5, None),
                                            (4, [3, 0, 4, 7])])
def test_mixed_lengths_gqa_match_torch_sdpa(window, windows):
    w = small_mixed(window=window, windows=windows)
    got = oracle.decode(problem_of(w))
    wof = (lambda b: windows[b]) if windows is not None else (lambda b: window)
    ref = sdpa_reference(w, wof)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_matches_pure_python_loops():
    w = make_workload(seq_lens=[6, 11], query_lens=[2, 1], num_q_heads=4,
                      num_kv_heads=2, head_dim=4, block_size=4, window=4,
                      dist="uniform", seed=5, scale=0.7)
    got = oracle.decode(problem_of(w))
    q = w.q.double().tolist()
    kc = w.k_cache.double().tolist()
    vc = w.v_cache.double().tolist()
    tok = 0
    for b in range(w.batch):
        S, L = int(w.seq_lens[b]), int(w.query_lens[b])
        for i in range(L):
            p = S - L + i
            for h in range(4):
                g = h // 2
                ts = [t for t in range(S) if p - 4 < t <= p]
                s = []
                for t in ts:
                    phys = int(w.block_tables[b, t // 4])
                    s.append(0.7 * sum(q[tok][h][x] * kc[phys][g][t % 4][x] for x in range(4)))
                m = max(s)
                e = [math.exp(x - m) for x in s]
                z = sum(e)
                for x in range(4):
                    ref = sum(e[j] / z * vc[int(w.block_tables[b, t // 4])][g][t % 4][x]
                              for j, t in enumerate(ts))
                    assert abs(got[tok, h, x] - ref) <= 1e-13
            tok += 1


def test_window_at_or_beyond_context_equals_unlimited():
    w = small_mixed()
    base = oracle.decode(problem_of(w, window=0))
    smax = int(w.seq_lens.max())
    for win in (smax, smax + 1, 10 ** 6):
        assert np.array_equal(oracle.decode(problem_of(w, window=win)), base)
    # per-row windows equal to each row's own context length
    per_row = w.seq_lens.tolist()
    assert np.array_equal(oracle.decode(problem_of(w, windows=per_row)), base)


def test_window_zero_is_full_causal():
    w = small_mixed()
    got = oracle.decode(problem_of(w, window=0))
    ref = sdpa_reference(w, lambda b: 0)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_window_one_returns_own_value_exactly():
    w = small_mixed(window=1)
    got = oracle.decode(problem_of(w))
    tok = 0
    G = w.num_q_heads // w.num_kv_heads
    for b in range(w.batch):
        S, L = int(w.seq_lens[b]), int(w.query_lens[b])
        for i in range(L):
            p = S - L + i
            phys = int(w.block_tables[b, p // w.block_size])
            for h in range(w.num_q_heads):
                v = w.v_cache[phys, h // G, p % w.block_size].double().numpy()
                assert np.array_equal(got[tok, h], v)
            tok += 1


def test_equal_keys_give_mean_of_visible_values():
    w = small_mixed(window=5)
    w.k_cache[:] = w.k_cache[0, 0, 0]          # every key identical
    got = oracle.decode(problem_of(w))
    tok = 0
    G = w.num_q_heads // w.num_kv_heads
    for b in range(w.batch):
        S, L = int(w.seq_lens[b]), int(w.query_lens[b])
        for i in range(L):
            p = S - L + i
            ts = range(max(0, p - 4), p + 1)
            for h in range(w.num_q_heads):
                vs = [w.v_cache[int(w.block_tables[b, t // w.block_size]), h // G,
                                t % w.block_size].double() for t in ts]
                ref = torch.stack(vs).mean(0).numpy()
                assert np.max(np.abs(got[tok, h] - ref)) <= 1e-14
            tok += 1


def test_two_visible_tokens_give_logistic_weights():
    # one row, two cached tokens, window 2: the last query token sees both;
    # weight of token 1 is 1 / (1 + exp(s0 - s1)).
    w = make_workload(seq_lens=[2], query_lens=[1], num_q_heads=1,
                      num_kv_heads=1, head_dim=8, block_size=16, window=2,
                      dist="uniform", seed=3, scale=0.9)
    pr = problem_of(w)
    got = oracle.decode(pr)[0, 0]
    q = w.q[0, 0].double()
    k = w.k_cache[int(w.block_tables[0, 0]), 0, :2].double()
    v = w.v_cache[int(w.block_tables[0, 0]), 0, :2].double()
    s0, s1 = (0.9 * (k @ q)).tolist()
    w1 = 1.0 / (1.0 + math.exp(s0 - s1))
    ref = ((1 - w1) * v[0] + w1 * v[1]).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-15
    wts = oracle.softmax_weights(pr, 0, 0, 0)
    assert abs(wts[1] - w1) <= 1e-15


def test_scale_is_applied_exactly():
    w = small_mixed()
    a = oracle.decode(problem_of(w))
    w2 = small_mixed()
    w2.q.mul_(2.0)                              # exact in bf16
    w2.scale = w.scale / 2.0
    b = oracle.decode(problem_of(w2))
    assert np.max(np.abs(a - b)) <= 1e-13
    w3 = small_mixed()
    w3.scale = w.scale * 3.0
    c = oracle.decode(problem_of(w3))
    assert np.max(np.abs(a - c)) > 1e-3         # the scale matters


def test_block_placement_does_not_matter():
    w = small_mixed(window=6)
    base = oracle.decode(problem_of(w))
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(w.num_blocks, generator=g)
    inv = torch.argsort(perm)
    w2 = small_mixed(window=6)
    w2.k_cache = w.k_cache[perm].clone()        # new slot j holds old block perm[j]
    w2.v_cache = w.v_cache[perm].clone()
    w2.block_tables = inv[w.block_tables.long()].to(torch.int32)
    assert np.array_equal(oracle.decode(problem_of(w2)), base)


def test_key_and_value_caches_are_not_interchangeable():
    w = small_mixed()
    base = oracle.decode(problem_of(w))
    w2 = small_mixed()
    w2.k_cache, w2.v_cache = w.v_cache.clone(), w.k_cache.clone()
    assert np.max(np.abs(oracle.decode(problem_of(w2)) - base)) > 1e-3


@pytest.mark.parametrize("window", [0, 7])
def test_split_k_invariance(window):
    w = small_mixed(window=window)
    pr = problem_of(w)
    base = oracle.decode(pr)
    nblk = int(math.ceil(int(w.seq_lens.max()) / w.block_size))
    for parts in (1, 2, 3, 7, nblk, 40):
        got = oracle.decode(pr, parts=parts)
        assert np.max(np.abs(got - base)) <= 1e-12, parts


def test_weights_sum_to_one_and_vanish_outside_range():
    w = small_mixed(window=6)
    pr = problem_of(w)
    lo, hi = oracle.visible_ranges(w.seq_lens.numpy(), w.query_lens.numpy(), 6)
    tok = 0
    for b in range(w.batch):
        for i in range(int(w.query_lens[b])):
            for h in range(w.num_q_heads):
                wts = oracle.softmax_weights(pr, b, i, h)
                assert abs(wts.sum() - 1.0) <= 1e-12
                assert np.all(wts[:lo[tok]] == 0) and np.all(wts[hi[tok]:] == 0)
                assert np.all(wts[lo[tok]:hi[tok]] > 0)
            tok += 1


def test_outputs_lie_in_convex_hull_of_visible_values():
    w = small_mixed(window=0)
    got = oracle.decode(problem_of(w))
    tok = 0
    G = w.num_q_heads // w.num_kv_heads
    for b in range(w.batch):
        S, L = int(w.seq_lens[b]), int(w.query_lens[b])
        k, v = dense_kv(w, b)
        for i in range(L):
            p = S - L + i
            for h in range(w.num_q_heads):
                vv = v[:p + 1, h // G].numpy()
                assert np.all(got[tok, h] <= vv.max(0) + 1e-12)
                assert np.all(got[tok, h] >= vv.min(0) - 1e-12)
            tok += 1


def test_golden_visible_ranges():
    rows = [list(map(int, ln.split())) for ln in open(GOLDEN)
            if ln.strip() and not ln.startswith("#")]
    assert rows
    for S, L, win, i, lo, hi in rows:
        los, his = oracle.visible_ranges([S], [L], win)
        assert (int(los[i]), int(his[i])) == (lo, hi), (S, L, win, i)


def test_visible_ranges_packing_and_per_row_windows():
    lo, hi = oracle.visible_ranges([300, 40, 7], [5, 1, 3], windows=[16, 0, 2])
    assert lo.tolist() == [280, 281, 282, 283, 284, 0, 3, 4, 5]
    assert hi.tolist() == [296, 297, 298, 299, 300, 40, 5, 6, 7]


def test_select_matches_full():
    w = small_mixed(window=3)
    pr = problem_of(w)
    full = oracle.decode(pr)
    sel = [(0, 0, 5), (1, 2, 0), (2, 4, 3), (3, 1, 1)]
    got = oracle.decode_select(pr, sel)
    qoff = np.concatenate([[0], np.cumsum(w.query_lens.numpy())])
    for j, (b, i, h) in enumerate(sel):
        assert np.array_equal(got[j], full[qoff[b] + i, h])


@pytest.mark.parametrize("bad", ["hq_not_multiple", "query_longer_than_seq",
                                 "negative_window", "table_out_of_range",
                                 "negative_row_window"])
def test_invalid_problems_are_rejected(bad):
    w = small_mixed()
    pr = problem_of(w)
    if bad == "hq_not_multiple":
        pr.hq = 5
    elif bad == "query_longer_than_seq":
        pr.query_lens = pr.query_lens.copy()
        pr.query_lens[0] = pr.seq_lens[0] + 1
    elif bad == "negative_window":
        pr.window = -1
    elif bad == "table_out_of_range":
        pr.block_tables = pr.block_tables.copy()
        pr.block_tables[0, 0] = pr.num_blocks
    elif bad == "negative_row_window":
        pr.windows = np.array([0, -2, 0, 0], dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.decode(pr)


def test_empty_query_rows_produce_no_outputs():
    w = make_workload(seq_lens=[5, 9, 3], query_lens=[0, 2, 0], num_q_heads=2,
                      num_kv_heads=1, head_dim=8, block_size=4, seed=2)
    got = oracle.decode(problem_of(w))
    assert got.shape == (2, 2, 8)
    ref = sdpa_reference(w, lambda b: 0)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_unreachable_blocks_match_brute_force():
    # A block is dead when no position in it is visible to any query token of
    # the row now or later (later tokens only move the window right): brute
    # force over every position of every leading block.
    rng = np.random.default_rng(4)
    for _ in range(300):
        bs = int(rng.choice([16, 32, 1024]))
        S = int(rng.integers(1, 6000))
        L = int(rng.integers(0, min(S, 6) + 1))
        w = int(rng.choice([0, 1, 5, 16, 100, 4096, int(rng.integers(1, 7000))]))
        got = int(oracle.unreachable_blocks([S], [L], bs, w)[0])
        want = 0
        if L > 0 and w > 0:
            for j in range((S + bs - 1) // bs):
                seen = False
                for p_ in range(S - L, S + 3):   # current tokens and a few later ones
                    lo = max(0, p_ + 1 - w)
                    if any(lo <= t <= p_ for t in range(j * bs, (j + 1) * bs)):
                        seen = True
                        break
                if seen:
                    break
                want += 1
        assert got == want, (S, L, w, bs)


def test_unreachable_blocks_on_the_gllm_batch():
    # 5-token chunk over 300 and a decode row over 40, 16-token blocks
    assert oracle.unreachable_blocks([300, 40], [5, 1], 16, 16).tolist() == [17, 1]
    assert oracle.unreachable_blocks([300, 40], [5, 1], 16, 100).tolist() == [12, 0]
    assert oracle.unreachable_blocks([300, 40], [5, 1], 16, 0).tolist() == [0, 0]
    assert oracle.unreachable_blocks([300, 40], [0, 1], 16, windows=[16, 4096]).tolist() == [0, 0]


def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert list(np.flatnonzero(nan)) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x38, 1.0), (0xB8, -1.0), (0x7E, 448.0), (0xFE, -448.0),
    (0x08, 2.0 ** -6), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),
    (0x3C, 1.5), (0x41, 2.25), (0x57, 15.0)])
def test_e4m3_closed_forms(code, value):
    # sign | 4 exponent bits (bias 7) | 3 mantissa bits; exponent 0 is subnormal
    got = oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0]
    assert got == value
    if code == 0x00:
        assert not math.copysign(1.0, oracle.e4m3_decode(np.array([0x80], np.uint8))[0]) > 0


def fp8_mixed(window=0, windows=None, seed=13, q_dtype="bf16", kv_dtype="fp8_e4m3"):
    return make_workload(seq_lens=[9, 23, 5, 31], query_lens=[1, 3, 5, 2],
                         num_q_heads=6, num_kv_heads=2, head_dim=16,
                         block_size=4, window=window, windows=windows,
                         dist="normal", seed=seed, scale=0.3, kv_dtype=kv_dtype,
                         q_dtype=q_dtype)


@pytest.mark.parametrize("window,windows", [(0, None), (5, None), (4, [3, 0, 4, 7])])
def test_fp8_caches_match_sdpa_on_dequantised_values(window, windows):
    w = fp8_mixed(window, windows)
    assert w.kv_fp8 and w.k_scale != w.v_scale
    got = oracle.decode(problem_of(w))
    wof = (lambda b: windows[b]) if windows is not None else (lambda b: window)
    ref = sdpa_reference(w, wof)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_fp8_scales_act_on_logits_and_output():
    w = fp8_mixed()
    base = problem_of(w)
    o = oracle.decode(base)
    args = (base.q, base.k_cache, base.v_cache, base.block_tables, base.seq_lens,
            base.query_lens)
    # v_scale is a factor on every output (a power of two keeps it exact)
    o2 = oracle.decode(oracle.Problem(*args, w.scale, k_scale=w.k_scale,
                                      v_scale=2 * w.v_scale))
    assert np.array_equal(o2, 2 * o)
    # k_scale enters only through the logits: k_scale*c is the same as scale*c
    o3 = oracle.decode(oracle.Problem(*args, w.scale * 1.7, k_scale=w.k_scale,
                                      v_scale=w.v_scale))
    o4 = oracle.decode(oracle.Problem(*args, w.scale, k_scale=w.k_scale * 1.7,
                                      v_scale=w.v_scale))
    assert np.max(np.abs(o3 - o4)) <= 1e-13
    assert np.max(np.abs(o3 - o)) > 1e-3


def test_fp8_split_k_invariance():
    w = fp8_mixed(window=7)
    pr = problem_of(w)
    o = oracle.decode(pr)
    for parts in (1, 2, 5):
        assert np.max(np.abs(oracle.decode(pr, parts=parts) - o)) <= 1e-13


@pytest.mark.parametrize("q_dtype,kv_dtype", [("fp8_e4m3", "bf16"), ("fp8_e4m3", "fp8_e4m3")])
def test_fp8_query_matches_sdpa_on_dequantised_values(q_dtype, kv_dtype):
    w = fp8_mixed(window=5, q_dtype=q_dtype, kv_dtype=kv_dtype)
    assert w.q_fp8 and w.q_scale > 0
    got = oracle.decode(problem_of(w))
    ref = sdpa_reference(w, lambda b: 5)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_fp8_query_scale_acts_on_the_logits():
    w = fp8_mixed(q_dtype="fp8_e4m3")
    pr = problem_of(w)
    args = (pr.q, pr.k_cache, pr.v_cache, pr.block_tables, pr.seq_lens, pr.query_lens)
    kw = dict(k_scale=w.k_scale, v_scale=w.v_scale)
    a = oracle.decode(oracle.Problem(*args, w.scale * 1.3, q_scale=w.q_scale, **kw))
    b = oracle.decode(oracle.Problem(*args, w.scale, q_scale=w.q_scale * 1.3, **kw))
    assert np.max(np.abs(a - b)) <= 1e-13


def random_pin_workload(seed):
    """Seeded random shapes for the SDPA pin: head_dim 8-256, block sizes 1-1024,
    GQA groups 1-8 over 1-3 kv heads, 1-5 rows of 1-600 tokens with 0-5
    query tokens, no window / one window / per-row windows, bf16 or FP8."""
    g = np.random.default_rng(700 + seed)
    B = int(g.integers(1, 6))
    S = [int(g.integers(1, 601)) for _ in range(B)]
    L = [int(min(s, g.integers(0, 6))) for s in S]
    if sum(L) == 0:
        L[0] = 1
    hkv = int(g.choice([1, 2, 3]))
    mode = g.choice(["none", "one", "rows"])
    window = int(g.choice([1, 3, 50])) if mode == "one" else 0
    windows = [int(g.choice([0, 1, 2, 17, 400])) for _ in range(B)] if mode == "rows" else None
    w = make_workload(seq_lens=S, query_lens=L, num_q_heads=hkv * int(g.choice([1, 2, 5, 8])),
                      num_kv_heads=hkv, head_dim=int(g.choice([8, 64, 128, 256])),
                      block_size=int(g.choice([1, 4, 16, 1024])), window=window,
                      windows=windows, dist=str(g.choice(["normal", "uniform"])),
                      seed=800 + seed, scale=float(g.uniform(0.05, 0.5)),
                      kv_dtype="fp8_e4m3" if g.random() < 0.3 else "bf16",
                      q_dtype="fp8_e4m3" if g.random() < 0.15 else "bf16")
    return w, (lambda b: windows[b]) if windows is not None else (lambda b: window)


@pytest.mark.parametrize("seed", range(24))
def test_random_shapes_match_torch_sdpa(seed):
    # the dense-gather SDPA pin over random shapes, windows and dtypes, and
    # the split-K form at a random partition count
    w, wof = random_pin_workload(seed)
    pr = problem_of(w)
    got = oracle.decode(pr)
    assert np.max(np.abs(got - sdpa_reference(w, wof))) <= 1e-12
    parts = int(np.random.default_rng(seed).integers(2, 9))
    assert np.max(np.abs(oracle.decode(pr, parts=parts) - got)) <= 1e-12
