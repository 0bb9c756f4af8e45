"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element.

Tolerance (from the method's stated bar for bf16 inputs with fp32 accumulation): max-abs
error <= 2e-2 and mean relative error <= 5e-3, the latter read as the ratio of L1 norms
sum|gpu - ref| / sum|ref| (elementwise relative error is ill-conditioned for outputs near 0).
The oracle consumes exactly the bf16-rounded (or fp32) values the kernel reads.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import prefix_shared_attention_b200 as bat
from workloads import (CONFIGS, RequestTable, device_tensors, gather_requests, host_tensors, make_table,
                       random_table, split_launches)

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_REL = 5e-3
LSE_ABS = 2e-2
# Guard rows around every output and LSE buffer: the kernels may write only inside the tensors
# they are given, so the guards must hold their sentinel afterwards (a stand-in for a memory
# checker, which is not available on the GPU pool).
GUARD_ROWS = 128
GUARD_VAL = -7.25


def dcode(dtype):
    return bat.BAT_BF16 if dtype == "bf16" else bat.BAT_FP32


def guarded(n_rows, row_shape, dtype, device):
    """A buffer of n_rows rows (filled with NaN, so an unwritten row shows) between GUARD_ROWS
    sentinel rows on each side; returns (whole buffer, view of the n_rows rows)."""
    buf = torch.full((n_rows + 2 * GUARD_ROWS,) + tuple(row_shape), float("nan"), dtype=dtype, device=device)
    buf[:GUARD_ROWS] = GUARD_VAL
    buf[GUARD_ROWS + n_rows:] = GUARD_VAL
    return buf, buf[GUARD_ROWS:GUARD_ROWS + n_rows]


def assert_guards(buf, n_rows, what):
    g = torch.cat([buf[:GUARD_ROWS].reshape(-1), buf[GUARD_ROWS + n_rows:].reshape(-1)])
    assert bool((g == GUARD_VAL).all()), f"{what}: a kernel wrote outside the tensor it was given"


def run_gpu(tab, xd, H, d, dtype, want_lse=True, scale=0.0, **plan_kw):
    """xd: dict of device tensors. Returns (out, lse) device tensors; checks that nothing was
    written into the guard rows around them."""
    T = xd["q"].shape[0]
    out_buf, out = guarded(T, xd["q"].shape[1:], xd["q"].dtype, xd["q"].device)
    n_lse = H * max(tab.T_suf, 1)
    if want_lse:
        lse_buf, lse_flat = guarded(n_lse, (), torch.float32, xd["q"].device)
        lse = lse_flat.view(H, max(tab.T_suf, 1))
    else:
        lse = None
    with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, H, d, dcode(dtype), **plan_kw) as plan:
        bat.bat_attention_forward(plan, xd["q"], xd["k_suf"], xd["v_suf"], xd["k_cache"], xd["v_cache"], out=out,
                                  lse=lse, scale=scale)
        st = bat.bat_get_device_status()
    assert st == bat.BAT_OK, bat.last_error()
    assert_guards(out_buf, T, "out")
    if want_lse:
        assert_guards(lse_buf, n_lse, "lse")
    return out, lse


def errors(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    diff = np.abs(gpu - ref)
    return float(diff.max()) if diff.size else 0.0, float(diff.sum() / max(np.abs(ref).sum(), 1e-30))


def assert_parity(out, lse, ref_o, ref_l, what=""):
    o = out.float().cpu().double().numpy()
    assert np.isfinite(o).all(), f"{what}: non-finite or unwritten output rows"
    mx, mr = errors(o, ref_o)
    assert mx <= MAX_ABS and mr <= MEAN_REL, f"{what}: max-abs {mx:.3g} (<= {MAX_ABS}), mean-rel {mr:.3g} (<= {MEAN_REL})"
    if lse is not None:
        l = lse.cpu().double().numpy()[:, :ref_l.shape[1]]
        lmx = float(np.abs(l - ref_l).max()) if l.size else 0.0
        assert lmx <= LSE_ABS, f"{what}: lse max-abs {lmx:.3g}"
    return mx, mr


def full_parity(tab, H, d, dtype, seed, scale=0.0, mutate=None, **plan_kw):
    x = host_tensors(tab, H, d, dtype, seed)
    if mutate:
        mutate(x)
    xd = {k: v.cuda() for k, v in x.items()}
    out, lse = run_gpu(tab, xd, H, d, dtype, scale=scale, **plan_kw)
    ref_o, ref_l = oracle.bipartite_attention(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"],
                                              tab.prefix_offsets, tab.suffix_offsets, tab.req_prefix,
                                              scale=scale if scale > 0 else None)
    return assert_parity(out, lse, ref_o, ref_l, f"H={H} d={d} {dtype} {plan_kw}")


# --------------------------------------------------------------------------------------
# small cases the oracle finishes in seconds: several tiles per request and a ragged tail

def test_tiny_config():
    spec = CONFIGS["tiny"]
    full_parity(make_table("tiny"), spec.H, spec.d, spec.dtype, spec.seed)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_bf16_ragged(d, seed):
    rng = np.random.default_rng(1000 + seed)
    tab = random_table(rng, P=3, R=7, max_prefix=600, max_suffix=500)
    full_parity(tab, 2, d, "bf16", seed)


@pytest.mark.parametrize("d", [32, 64, 128])
def test_fp32_ragged(d):
    rng = np.random.default_rng(2000 + d)
    tab = random_table(rng, P=2, R=5, max_prefix=300, max_suffix=260)
    full_parity(tab, 2, d, "fp32", d)


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("bf16", 128), ("fp32", 64)])
@pytest.mark.parametrize("chunk", [1, 3])
def test_forced_split_merge(dtype, d, chunk):
    rng = np.random.default_rng(3000 + d + chunk)
    tab = random_table(rng, P=3, R=6, max_prefix=700, max_suffix=400)
    full_parity(tab, 2, d, dtype, 7, split_mode=2, split_chunk_tiles=chunk)


@pytest.mark.parametrize("d", [64, 128])
def test_edge_lengths(d):
    # empty prefix, Ls = 1, exact tile multiples, one past a multiple, a prefix read by one
    # request, a request with no prefix, an unreferenced prefix, an empty suffix.
    tab = RequestTable(np.array([0, 128, 129, 1, 640]), np.array([0, 1, 2, 3, -1, 1, 2, 1, 1], np.int32),
                       np.array([1, 128, 129, 255, 256, 1, 0, 384, 3]))
    full_parity(tab, 3, d, "bf16", 11)


@pytest.mark.parametrize("d", [64, 128])
def test_short_key_tiles(d):
    # Key tiles with at most 32 or 64 valid keys (short prefixes and ragged stream ends), for
    # which the d = 64 kernel computes only the first 64 key columns; the 63-key prefix
    # carries the row maximum, so a rescale happens on a short tile.
    pre = np.array([1, 31, 32, 33, 63, 64, 65, 96])
    tab = RequestTable(pre, np.array([0, 1, 2, 3, 4, 5, 6, 7, 5, 4], np.int32),
                       np.array([64, 160, 192, 129, 191, 33, 64, 200, 130, 63]))

    def mutate(x):
        x["k_cache"][int(pre[:4].sum()):int(pre[:5].sum())] *= 8.0

    full_parity(tab, 2, d, "bf16", 21, mutate=mutate)


@pytest.mark.parametrize("d", [64, 128])
def test_explicit_scale(d):
    rng = np.random.default_rng(77)
    tab = random_table(rng, P=2, R=4, max_prefix=300, max_suffix=300)
    full_parity(tab, 2, d, "bf16", 5, scale=0.05)


@pytest.mark.parametrize("d", [64, 128])
def test_running_max_rescale_path(d):
    # Later key tiles carry much larger scores, so the running maximum jumps by far more than
    # the lazy-rescale threshold several times within one row.
    tab = RequestTable(np.array([640]), np.array([0, 0, -1], np.int32), np.array([300, 129, 260]))

    def mutate(x):
        x["k_cache"][256:384] *= 6.0
        x["k_cache"][512:] *= 12.0
        x["k_suf"][200:300] *= 20.0
        x["k_suf"][429 + 130:] *= 16.0

    full_parity(tab, 2, d, "bf16", 13, mutate=mutate)


def test_gpu_role_swap_invariant():
    """Invariant (1) on the GPU: cache the user block and run the items as suffix, then the
    other way round; both give the monolithic attention rows within the parity bar."""
    rng = np.random.default_rng(5)
    H, d, n = 2, 64, 4
    ul, il = rng.integers(50, 300, n), rng.integers(50, 300, n)
    g = torch.Generator().manual_seed(5)
    toks = {k: [torch.randn(ul[i] + il[i], H, d, generator=g).bfloat16() for i in range(n)] for k in "qkv"}
    results = {}
    for user_prefix in (True, False):
        pre = [slice(0, ul[i]) if user_prefix else slice(ul[i], ul[i] + il[i]) for i in range(n)]
        suf = [slice(ul[i], ul[i] + il[i]) if user_prefix else slice(0, ul[i]) for i in range(n)]
        cat = lambda k, sl: torch.cat([toks[k][i][sl[i]] for i in range(n)]).cuda()
        tab = RequestTable(np.array([s.stop - s.start for s in pre]), np.arange(n),
                           np.array([s.stop - s.start for s in suf]))
        xd = dict(q=cat("q", suf), k_suf=cat("k", suf), v_suf=cat("v", suf), k_cache=cat("k", pre), v_cache=cat("v", pre))
        out, _ = run_gpu(tab, xd, H, d, "bf16", want_lse=False)
        results[user_prefix] = (tab, out.float().cpu().double().numpy())
    for i in range(n):
        for h in range(H):
            Q, K, V = (toks[k][i][:, h].double().numpy() for k in "qkv")
            mono, _ = oracle.attend(Q, K, V, 1 / math.sqrt(d))
            tab_u, ou = results[True]
            tab_i, oi = results[False]
            item_rows = slice(tab_u.suffix_offsets[i], tab_u.suffix_offsets[i + 1])
            user_rows = slice(tab_i.suffix_offsets[i], tab_i.suffix_offsets[i + 1])
            for got, want in ((ou[item_rows, h], mono[ul[i]:]), (oi[user_rows, h], mono[:ul[i]])):
                mx, mr = errors(got, want)
                assert mx <= MAX_ABS and mr <= MEAN_REL


def test_prefix_kv_build_is_exact():
    torch.manual_seed(3)
    H, d = 4, 64
    lens = [5, 0, 130, 64]
    src_off = np.concatenate([[0], np.cumsum(lens)])
    k_src = torch.randn(int(src_off[-1]), H, d, device="cuda").bfloat16()
    v_src = torch.randn_like(k_src)
    dst_off = np.array([300, 7, 20, 150])            # scattered into a larger pool
    kc = torch.zeros(400, H, d, device="cuda", dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    bat.bat_prefix_kv_build(k_src, v_src, src_off, dst_off, kc, vc)
    torch.cuda.synchronize()
    for i, L in enumerate(lens):
        a, b = int(src_off[i]), int(src_off[i + 1])
        assert torch.equal(kc[dst_off[i]:dst_off[i] + L], k_src[a:b])
        assert torch.equal(vc[dst_off[i]:dst_off[i] + L], v_src[a:b])
    untouched = torch.ones(400, dtype=torch.bool)
    for i, L in enumerate(lens):
        untouched[dst_off[i]:dst_off[i] + L] = False
    assert (kc[untouched.cuda()] == 0).all()


def test_wait_timeout_reports_and_context_survives():
    rng = np.random.default_rng(9)
    tab = random_table(rng, P=2, R=4, max_prefix=500, max_suffix=400)
    x = host_tensors(tab, 2, 128, "bf16", 9)
    xd = {k: v.cuda() for k, v in x.items()}
    bat.bat_set_wait_timeout_ns(1)   # every wait that is not already satisfied runs out at once
    try:
        with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, 2, 128) as plan:
            out = torch.empty_like(xd["q"])
            bat.bat_attention_forward(plan, xd["q"], xd["k_suf"], xd["v_suf"], xd["k_cache"], xd["v_cache"], out=out)
            st = bat.bat_get_device_status()
    finally:
        bat.bat_set_wait_timeout_ns(0)
    # With a 1 ns limit the first wait whose phase has not completed yet expires (the softmax
    # waits for an S that the tensor core cannot have finished when it first looks), so the
    # abort path must have run and reported.
    assert st == bat.BAT_ERR_TIMEOUT, f"expected BAT_ERR_TIMEOUT, got {st}: {bat.last_error()}"
    # The context stays usable and the next run is correct.
    full_parity(tab, 2, 128, "bf16", 9)
    assert bat.bat_get_device_status() == bat.BAT_OK


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("bf16", 128), ("fp32", 64)])
@pytest.mark.parametrize("split", [0, 2])
def test_nan_neighbour_rows(dtype, d, split):
    """Rows that a tile window reaches beyond its segment may hold anything, NaN included:
    cache slots reserved but not yet built (allocated uninitialised), or another request's
    garbage tokens.  Masked keys must weigh exactly 0 there, so every other request's output
    stays exact.  Lead page (Bat), section "This paper's idea": the prefix K/V is computed once
    and kept in a pool that many requests read, so one bad slot must not reach them."""
    # Pool: referenced prefixes (even ids) interleaved with unreferenced NaN slots (odd ids),
    # one NaN slot after the last prefix; lengths end inside a 16-key step.
    pre = np.array([37, 21, 201, 7, 99, 300, 130, 50, 1, 19])
    nan_pre = [1, 3, 5, 7, 9]
    req = np.array([0, 0, 2, 4, 6, 2, -1, 4, 6, 0, 8, 2], np.int32)
    suf = np.array([45, 130, 77, 1, 257, 19, 100, 128, 33, 200, 70, 131])
    poisoned = [5, 8]                       # requests whose own q/k/v rows are NaN
    tab = RequestTable(pre, req, suf)
    po, so = tab.prefix_offsets, tab.suffix_offsets

    def mutate(x):
        for p in nan_pre:
            x["k_cache"][po[p]:po[p + 1]] = float("nan")
            x["v_cache"][po[p]:po[p + 1]] = float("nan")
        for r in poisoned:
            for k in ("q", "k_suf", "v_suf"):
                x[k][so[r]:so[r + 1]] = float("nan")

    H = 2
    x = host_tensors(tab, H, d, dtype, 31)
    mutate(x)
    xd = {k: v.cuda() for k, v in x.items()}
    out, lse = run_gpu(tab, xd, H, d, dtype, split_mode=split, split_chunk_tiles=1 if split else 0)
    ref_o, ref_l = oracle.bipartite_attention(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"], po, so,
                                              tab.req_prefix)
    keep = np.ones(tab.T_suf, bool)
    for r in poisoned:
        keep[so[r]:so[r + 1]] = False
    assert np.isfinite(ref_o[keep]).all()
    o = out.float().cpu().double().numpy()
    assert np.isfinite(o[keep]).all(), "a NaN in a masked row leaked into another request's output"
    mx, mr = errors(o[keep], ref_o[keep])
    assert mx <= MAX_ABS and mr <= MEAN_REL, (mx, mr)
    lmx = float(np.abs(lse.cpu().double().numpy()[:, keep] - ref_l[:, keep]).max())
    assert lmx <= LSE_ABS, lmx


# --------------------------------------------------------------------------------------
# named configurations at full size, in the launch configuration the bench times;
# a seeded sample of requests is checked against the oracle

def sampled_parity(name, n_sample, launch=None, n_launches=1, seed=123):
    spec = CONFIGS[name]
    tab = make_table(name)
    if n_launches > 1:
        tab = split_launches(tab, n_launches)[launch]
    xd = device_tensors(tab, spec.H, spec.d, spec.dtype, spec.seed + 17)
    out, lse = run_gpu(tab, xd, spec.H, spec.d, spec.dtype)
    rng = np.random.default_rng(seed)
    reqs = np.sort(rng.choice(tab.R, size=min(n_sample, tab.R), replace=False))
    reqs = reqs[tab.suffix_len[reqs] > 0]
    sub, host, rows = gather_requests(tab, xd, reqs, out=out)
    lse_rows = lse[:, torch.from_numpy(rows).cuda()].cpu()
    ref_o, ref_l = oracle.bipartite_attention(host["q"], host["k_suf"], host["v_suf"], host["k_cache"],
                                              host["v_cache"], sub.prefix_offsets, sub.suffix_offsets, sub.req_prefix)
    res = assert_parity(host["out"], lse_rows, ref_o, ref_l, name)
    del xd, out, lse
    torch.cuda.empty_cache()
    return res


def test_user_as_prefix_full():
    sampled_parity("user-as-prefix", 512)     # every request


def test_item_as_prefix_sampled():
    sampled_parity("item-as-prefix", 256)


def test_long_user_history_sampled():
    sampled_parity("long-user-history", 16)


def mixed_sample(sub_tab, per_kind, rng):
    """Requests of one launch to check: `per_kind` of each prefix kind (user block cached /
    item block cached), drawn at random, plus the heaviest request of the launch (longest
    prefix + suffix: the deepest key stream and rescale chain)."""
    Lp = sub_tab.prefix_len_of_request()
    pick = [int(np.argmax(Lp + sub_tab.suffix_len))]
    for k in (0, 1):
        idx = np.flatnonzero(sub_tab.kind == k)
        pick += [int(i) for i in rng.choice(idx, size=min(per_kind, len(idx)), replace=False)]
    return np.unique(np.array(pick, np.int64))


def test_mixed_sampled_every_launch():
    """The mixed batch in the launch configuration the bench times (8 request-disjoint launches
    over one resident prefix cache): from every launch, 16 user-prefix and 16 item-prefix
    requests plus the launch's heaviest request, 264 in all, against the oracle."""
    free, _ = torch.cuda.mem_get_info()
    if free < 150e9:
        pytest.skip(f"needs ~140 GB free device memory, {free / 1e9:.0f} GB free")
    name = "mixed"
    spec = CONFIGS[name]
    tab = make_table(name)
    parts = split_launches(tab, 8)
    cache = device_tensors(tab, spec.H, spec.d, spec.dtype, spec.seed + 17, which=("k_cache", "v_cache"))
    rng = np.random.default_rng(123)
    checked = 0
    for i, part in enumerate(parts):
        xd = dict(cache)
        xd.update(device_tensors(part, spec.H, spec.d, spec.dtype, spec.seed + 100 + i, which=("q", "k_suf", "v_suf")))
        out, lse = run_gpu(part, xd, spec.H, spec.d, spec.dtype)
        reqs = mixed_sample(part, 16, rng)
        sub, host, rows = gather_requests(part, xd, reqs, out=out)
        lse_rows = lse[:, torch.from_numpy(rows).cuda()].cpu()
        ref_o, ref_l = oracle.bipartite_attention(host["q"], host["k_suf"], host["v_suf"], host["k_cache"],
                                                  host["v_cache"], sub.prefix_offsets, sub.suffix_offsets,
                                                  sub.req_prefix)
        assert_parity(host["out"], lse_rows, ref_o, ref_l, f"{name} launch {i}")
        checked += len(reqs)
        del xd, out, lse
        torch.cuda.empty_cache()
    assert checked >= 8 * 33


# --------------------------------------------------------------------------------------
# prefix-side step: the prefix tokens' own outputs, plus the K/V packed into the pool

@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("bf16", 128), ("fp32", 32)])
def test_prefix_side_step(dtype, d):
    lens = [0, 1, 63, 128, 129, 300, 517] if dtype == "bf16" else [0, 1, 40, 129]
    H = 2
    tab = RequestTable(np.zeros(0, np.int64), np.full(len(lens), -1), np.array(lens))
    x = host_tensors(tab, H, d, dtype, 77)
    q, k, v = (x[n].cuda() for n in ("q", "k_suf", "v_suf"))
    so = tab.suffix_offsets
    # Pack into a pool laid out in reverse prefix order (gaps of 3 rows between prefixes).
    dst, pos = np.zeros(len(lens), np.int64), 0
    for i in reversed(range(len(lens))):
        dst[i] = pos
        pos += lens[i] + 3
    kc = torch.zeros((pos, H, d), dtype=k.dtype, device="cuda")
    vc = torch.zeros_like(kc)
    lse = torch.full((H, max(tab.T_suf, 1)), float("nan"), device="cuda")
    out = bat.prefix_build(q, k, v, so, dst, kc, vc, lse=lse)
    assert bat.bat_get_device_status() == bat.BAT_OK, bat.last_error()
    for i, L in enumerate(lens):
        assert torch.equal(kc[dst[i]:dst[i] + L], k[so[i]:so[i + 1]]), f"K of prefix {i} not packed exactly"
        assert torch.equal(vc[dst[i]:dst[i] + L], v[so[i]:so[i + 1]]), f"V of prefix {i} not packed exactly"
    ref_o, ref_l = oracle.prefix_side_attention(x["q"].double().numpy(), x["k_suf"].double().numpy(),
                                                x["v_suf"].double().numpy(), so)
    assert_parity(out, lse, ref_o, ref_l, f"prefix side {dtype} d={d}")
