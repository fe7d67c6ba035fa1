"""GPU parity of the paged, ragged cache: slots of different lengths whose quantized
tokens live in pages of one pool.  Every slot is a KIVI cache of its own, so the
oracle is one single-sequence oracle cache per slot, fed the same seeded inputs.
Codes, scales and zeros (gathered through the page table) must match bit for bit;
outputs |gpu - ref| <= 2e-3 + 1e-2 |ref|; inactive and empty slots give zeros."""
import numpy as np
import pytest
import torch

from bit_kv_cache_22_b200 import kvq
from bit_kv_cache_22_b200 import workloads as wl

import kvq_testlib as tl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def new_paged(w: wl.Workload, page_tokens: int, capacity: int, num_pages=None) -> kvq.PagedKVQCache:
    return kvq.PagedKVQCache(w.B, w.Hq, w.Hkv, w.d, w.G, w.Gv, w.R, w.bits, w.symmetric,
                             tl.torch_dtype(w), capacity, page_tokens, num_pages, "cuda")


def paged_packed(cache: kvq.PagedKVQCache, b: int, Tq: int) -> dict:
    """Slot b's quantized tokens gathered from its pages, in the oracle's array shapes."""
    g = cache.geom
    Hkv, P = g.kv_heads, cache.page_tokens
    rows = [pg * Hkv + h for h in range(Hkv) for pg in cache.pages[b]]
    n = len(cache.pages[b])

    def gather(t, per_token_axis_len):
        x = t[rows].reshape(Hkv, n, *t.shape[1:])
        return x.reshape(Hkv, n * t.shape[1], *t.shape[2:])[:, :per_token_axis_len]

    words = Tq * g.head_dim * g.bits // 32
    out = dict(Kc=gather(cache.k_codes, words).cpu().numpy().view(np.uint32),
               Vc=gather(cache.v_codes, words).cpu().numpy().view(np.uint32),
               Ks=gather(cache.k_scales, Tq // g.group_k).cpu().numpy(),
               Vs=gather(cache.v_scales, Tq).cpu().numpy())
    if cache.k_zeros is not None:
        out["Kz"] = gather(cache.k_zeros, Tq // g.group_k).cpu().numpy()
        out["Vz"] = gather(cache.v_zeros, Tq).cpu().numpy()
    return out


class Episode:
    """A paged GPU cache and one oracle cache per active slot, stepped together."""

    def __init__(self, w: wl.Workload, lens, page_tokens: int, steps: int, num_pages=None,
                 shuffle_pages=False):
        self.w, self.steps = w, steps
        cap = -(-(max(x for x in lens if x is not None) + steps + 64) // page_tokens) * page_tokens
        self.cache = new_paged(w, page_tokens, cap, num_pages)
        if shuffle_pages:   # hand pages out in a scrambled order
            rng = np.random.default_rng(7)
            rng.shuffle(self.cache.free_pages)
        self.refs = [None] * w.B
        self.tK, self.tV, self.tQ = wl.decode_bits(w, steps=steps)
        for b, T in enumerate(lens):
            if T is not None:
                self.prefill(b, T, b)

    def prefill(self, b: int, T: int, seed_slot: int):
        w = self.w
        XK, XV = wl.prefill_bits(w, bs=[seed_slot], T=T)
        self.cache.prefill(b, tl.to_dev(XK[0], w), tl.to_dev(XV[0], w))
        ref = tl.new_oracle(w, B=1)
        ref.prefill(XK, XV)
        self.refs[b] = ref
        self.check_codes(b)

    def release(self, b: int):
        self.cache.release(b)
        self.refs[b] = None

    def check_codes(self, b: int):
        ref = self.refs[b]
        tl.assert_codes_equal(paged_packed(self.cache, b, ref.Tq), ref.packed(), self.w.symmetric)
        assert self.cache.seq_len(b) == ref.Tq + ref.r

    def append(self, s: int):
        w = self.w
        self.cache.append(tl.to_dev(self.tK[s], w), tl.to_dev(self.tV[s], w))
        for b, ref in enumerate(self.refs):
            if ref is not None:
                flushes = ref.flushes
                ref.append(self.tK[s][b:b + 1], self.tV[s][b:b + 1])
                if ref.flushes != flushes:
                    self.check_codes(b)

    def decode_and_check(self, s: int, what=""):
        w = self.w
        out = self.cache.decode_attention(tl.to_dev(self.tQ[s], w)).cpu().numpy()
        for b, ref in enumerate(self.refs):
            if ref is None or ref.Tq + ref.r == 0:
                assert not out[b].any(), f"{what} slot {b}: an empty slot must give zeros"
            else:
                tl.assert_close(out[b:b + 1], ref.decode(self.tQ[s][b:b + 1]), f"{what} step {s} slot {b}")
        return out


# (name, workload changes, slot lengths (None = inactive), page tokens): the tensor-core kernel
# with 1, 2 and 4 query heads per kv head, 4-bit groups of 128, the CUDA-core kernel (16-token
# key groups; 8 query heads per kv head), the symmetric variant
CASES = [
    ("tiny", dict(B=6, steps=0), [0, 5, 32, 97, None, 200], 64),
    ("llama7b", dict(B=4, Hq=2, Hkv=2), [300, 0, 1000, 133], 128),
    ("gqa8b", dict(B=5, Hq=8, Hkv=2), [700, None, 1, 128, 2100], 256),
    ("gqa8b", dict(B=4, Hq=4, Hkv=2, Gv=64), [129, 640, 64, 900], 128),
    ("stream2", dict(B=4, Hq=4, Hkv=2, G=16, Gv=16, R=64), [40, 700, None, 300], 64),
    ("stream2", dict(B=3, Hq=16, Hkv=2, d=64), [500, 260, 3], 128),
    ("stream4sym", dict(B=3, Hq=8, Hkv=2), [256, 77, 600], 128),
]


@pytest.mark.parametrize("name,changes,lens,P", CASES)
def test_paged_ragged_episode_matches_oracle(name, changes, lens, P):
    base = wl.WORKLOADS[name]
    w = base.replace(**{k: v for k, v in changes.items() if k != "steps"})
    steps = w.R + 9
    ep = Episode(w, lens, P, steps)
    ep.decode_and_check(0, "after prefill")
    for s in range(steps):
        ep.append(s)
        if s % 5 == 0 or s == steps - 1:
            ep.decode_and_check(s, name)
    # a slot ends and another prompt takes it (its pages are reused)
    b = next(i for i, x in enumerate(lens) if x is not None)
    ep.release(b)
    ep.decode_and_check(steps - 1, "after release")
    ep.prefill(b, 2 * w.R + 11, seed_slot=w.B + 1)
    ep.decode_and_check(steps - 1, "after re-prefill")
    ep.cache.check_device()


def test_paged_uniform_lengths_equal_the_contiguous_cache():
    """Same lengths in every slot: the paged kernels give the contiguous cache's outputs."""
    w = wl.WORKLOADS["gqa8b"].replace(B=3, Hq=8, Hkv=2, T=3 * 128 + 40, steps=20)
    XK, XV = wl.prefill_bits(w)
    tK, tV, tQ = wl.decode_bits(w)
    flat = tl.new_cache(w)
    flat.prefill_quantize(tl.to_dev(XK, w), tl.to_dev(XV, w))
    paged = new_paged(w, 128, 1024)
    rng = np.random.default_rng(3)
    rng.shuffle(paged.free_pages)
    for b in range(w.B):
        paged.prefill(b, tl.to_dev(XK[b], w), tl.to_dev(XV[b], w))
    for s in range(w.steps):
        flat.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        paged.append(tl.to_dev(tK[s], w), tl.to_dev(tV[s], w))
        a = flat.decode_attention(tl.to_dev(tQ[s], w))
        p = paged.decode_attention(tl.to_dev(tQ[s], w))
        if flat.splits() == paged.splits():
            assert torch.equal(a, p), f"step {s}"
        else:
            tl.assert_close(p.cpu().numpy(), a.cpu().numpy().astype(np.float64), f"step {s}")


def test_page_order_does_not_change_the_result():
    """Pages handed out in scrambled order give bit-identical outputs and codes."""
    w = wl.WORKLOADS["gqa8b"].replace(B=3, Hq=8, Hkv=2)
    lens = [900, 140, 520]
    a = Episode(w, lens, 128, 40)
    b = Episode(w, lens, 128, 40, shuffle_pages=True)
    assert a.cache.pages != b.cache.pages
    for s in range(40):
        a.append(s)
        b.append(s)
    oa = a.cache.decode_attention(tl.to_dev(a.tQ[-1], w))
    ob = b.cache.decode_attention(tl.to_dev(b.tQ[-1], w))
    assert torch.equal(oa, ob)


def test_all_slots_inactive_or_empty_give_zeros():
    w = wl.WORKLOADS["tiny"].replace(B=3)
    cache = new_paged(w, 64, 256)
    q = torch.randn(w.B, w.Hq, w.d, device="cuda").to(torch.float16)
    assert not cache.decode_attention(q).any()
    cache.prefill(1, torch.zeros(w.Hkv, 0, w.d, dtype=torch.float16, device="cuda"),
                  torch.zeros(w.Hkv, 0, w.d, dtype=torch.float16, device="cuda"))
    assert cache.seq_len(1) == 0 and cache.seq_len(0) == -1
    assert not cache.decode_attention(q).any()
    cache.check_device()


def test_page_outside_the_pool_is_reported_not_followed():
    """A page-table entry outside the pool: the kernels touch page 0 instead and raise the
    status bit that check_device reports (no out-of-bounds access)."""
    w = wl.WORKLOADS["gqa8b"].replace(B=2, Hq=8, Hkv=2)
    ep = Episode(w, [300, 200], 128, 4)
    ep.cache.check_device()
    ep.cache.page_table[0, 1] = ep.cache.num_pages + 5       # a page the pool does not have
    ep.cache.decode_attention(tl.to_dev(ep.tQ[0], w))
    torch.cuda.synchronize()
    with pytest.raises(kvq.KVQError):
        ep.cache.check_device()
    ep.cache.check_device()                                 # the word was cleared


def test_paged_errors():
    w = wl.WORKLOADS["tiny"].replace(B=2)
    cache = new_paged(w, 64, 128)
    X = torch.zeros(w.Hkv, 70, w.d, dtype=torch.float16, device="cuda")
    cache.prefill(0, X, X)
    with pytest.raises(kvq.KVQError):
        cache.prefill(0, X, X)                       # active slot
    big = torch.zeros(w.Hkv, 200, w.d, dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KVQError):
        cache.prefill(1, big, big)                   # beyond capacity
    t = torch.zeros(w.B, w.Hkv, w.d, dtype=torch.float16, device="cuda")
    for _ in range(160 - 70 - 1):                   # the flush at 128 tokens fits capacity 128
        cache.append(t, t)
    assert cache.seq_len(0) == 159
    with pytest.raises(kvq.KVQError):
        cache.append(t, t)                           # the flush at 160 would pass it
    assert cache.seq_len(0) == 159
    cache.check_device()
