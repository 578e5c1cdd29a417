"""CPU tests of the C ABI: the library loads, exports what the header declares,
rejects bad arguments before any launch, and its causal block rule matches the
brute-force mask.  No compute call is made (there may be no GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

from causal_prefill_attention_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "prefill.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*((?:prefill|paged|qkv|kv|attn)_[a-z_0-9]+)\s*\(", src,
                                 flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert "prefill_attn" in names and "prefill_attn_chunked" in names and "paged_decode_attn" in names
    for name in names:
        assert hasattr(lib, name), name
    assert set(_lib.EXPORTED) <= set(names)


def test_status_strings(lib):
    for s in range(9):
        assert _lib.status_string(s)
    assert _lib.status_string(99) == "unknown status"


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _call(lib, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, total=128, cu=FAKE, num_seqs=1, max_seqlen=128, H=4, G=4, D=128,
             scale=0.088, out=FAKE, cache=FAKE, nb=8, bt=FAKE, mbps=8, bs=16, status=None, stream=None)
    a.update(over)
    return lib.prefill_attn(a["q"], a["k"], a["v"], a["total"], a["cu"], a["num_seqs"], a["max_seqlen"], a["H"],
                            a["G"], a["D"], a["scale"], a["out"], a["cache"], a["nb"], a["bt"], a["mbps"], a["bs"],
                            a["status"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(cu=None), 1), (dict(bt=None), 1), (dict(cache=None), 1),
    (dict(H=6, G=4), 2), (dict(G=0), 2), (dict(total=-1), 2),
    (dict(D=96), 3), (dict(D=256), 3), (dict(bs=8), 3), (dict(bs=24), 3),
    (dict(scale=0.0), 3), (dict(scale=float("nan")), 3), (dict(scale=float("inf")), 3), (dict(scale=-1.0), 3),
    (dict(max_seqlen=129), 4), (dict(nb=0), 4), (dict(mbps=0), 4),
    (dict(q=FAKE + 8), 7), (dict(out=FAKE + 2), 7),
])
def test_host_validation_rejects_before_launch(lib, over, code):
    assert _call(lib, **over) == code


def test_empty_call_is_a_noop(lib):
    assert _call(lib, total=0) == 0
    assert _call(lib, num_seqs=0) == 0


def test_chunked_validation(lib):
    P = FAKE
    args = [P, P, P, 512, P, P, 1, 512, 7680, 32, 8, 128, 0.088, P, P, 512, P, 512, 16, None, None]
    a = list(args)
    a[5] = None  # context_lens
    assert lib.prefill_attn_chunked(*a) == 1
    a = list(args)
    a[8] = 8193  # the context bound alone exceeds the table
    assert lib.prefill_attn_chunked(*a) == 4
    a = list(args)
    a[7] = 8193  # the chunk bound alone exceeds the table
    assert lib.prefill_attn_chunked(*a) == 4


# ---------------------------------------------------------------- P11: block rule vs brute force
def _brute_visible(ctx, n):
    """visible[a, p] for chunk rows a < n and absolute key positions p < ctx + n."""
    a = np.arange(n)[:, None]
    p = np.arange(ctx + n)[None, :]
    return p <= ctx + a


@pytest.mark.parametrize("bm,bn", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_block_rule_matches_brute_force_mask(lib, bm, bn):
    rng = np.random.default_rng(5)
    cases = [(0, n) for n in (1, 2, 3, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 256, 300)]
    cases += [(int(c), int(n)) for c, n in zip(rng.integers(0, 400, 40), rng.integers(1, 300, 40))]
    cases += [(128, 128), (512, 512), (130, 5), (1, 1)]
    for ctx, n in cases:
        vis = _brute_visible(ctx, n)
        covered = np.zeros_like(vis, dtype=np.int32)
        for qb in range(-(-n // bm)):
            rows = np.arange(qb * bm, min(qb * bm + bm, n))
            nkv = _lib.num_kv_blocks(qb, ctx, n, bm, bn)
            for j in range(nkv):
                kind, lim, kb = _lib.kv_block_rule(qb, j, ctx, n, bm, bn)
                assert kind in (0, 1)
                for r_i, a in enumerate(rows):
                    r = a - qb * bm
                    cols = kb + np.arange(bn)
                    in_range = cols < ctx + n
                    want = np.zeros(bn, dtype=bool)
                    want[in_range] = vis[a, cols[in_range]]
                    # prefix blocks stop at ctx; chunk blocks never include prefix columns
                    if j < -(-ctx // bn):
                        want &= cols < ctx
                    got = np.arange(bn) < lim[r]
                    assert np.array_equal(got, want), (ctx, n, qb, j, a)
                    if kind == 0:
                        assert want.all()
                    covered[a, cols[got]] += 1
            assert _lib.kv_block_rule(qb, nkv, ctx, n, bm, bn)[0] == -1
        # every visible pair is covered by exactly one issued block; no invisible pair is
        assert np.array_equal(covered, vis.astype(np.int32)), (ctx, n)


# ---------------------------------------------------------------- block rule under a sliding window
def _brute_band(ctx, n, window):
    """visible[a, p]: chunk row a (absolute position ctx + a) sees key p iff
    ctx + a - window < p <= ctx + a."""
    a = np.arange(n)[:, None]
    p = np.arange(ctx + n)[None, :]
    return (p <= ctx + a) & (p > ctx + a - window)


@pytest.mark.parametrize("bm,bn", [(128, 128), (64, 64), (128, 64)])
def test_window_block_rule_matches_brute_force_band(lib, bm, bn):
    rng = np.random.default_rng(6)
    cases = [(0, 300, w) for w in (1, 2, 63, 64, 65, 127, 128, 129, 200, 299, 300, 1000)]
    cases += [(200, 300, w) for w in (1, 50, 128, 201, 260, 500)]
    cases += [(int(c), int(n), int(w)) for c, n, w in
              zip(rng.integers(0, 500, 40), rng.integers(1, 400, 40), rng.integers(1, 600, 40))]
    for ctx, n, window in cases:
        vis = _brute_band(ctx, n, window)
        covered = np.zeros_like(vis, dtype=np.int32)
        for qb in range(-(-n // bm)):
            rows = np.arange(qb * bm, min(qb * bm + bm, n))
            nkv = _lib.num_kv_blocks(qb, ctx, n, bm, bn)
            first = _lib.first_kv_block(qb, ctx, n, window, bm, bn)
            assert 0 <= first < nkv
            for j in range(first, nkv):
                kind, lo, lim, kb = _lib.kv_block_rule_window(qb, j, ctx, n, window, bm, bn)
                assert kind in (0, 1)
                any_visible = False
                for a in rows:
                    r = a - qb * bm
                    cols = kb + np.arange(bn)
                    in_range = cols < ctx + n
                    want = np.zeros(bn, dtype=bool)
                    want[in_range] = vis[a, cols[in_range]]
                    if j < -(-ctx // bn):
                        want &= cols < ctx
                    got = (np.arange(bn) >= lo[r]) & (np.arange(bn) < lim[r])
                    assert np.array_equal(got, want), (ctx, n, window, qb, j, a)
                    if kind == 0:
                        assert want.all()
                    any_visible |= bool(want.any())
                    covered[a, cols[got]] += 1
                if j == first:
                    assert any_visible, "the first issued block holds a visible pair"
            assert _lib.kv_block_rule_window(qb, first - 1, ctx, n, window, bm, bn)[0] == -1 or first == 0
            assert _lib.kv_block_rule_window(qb, nkv, ctx, n, window, bm, bn)[0] == -1
        assert np.array_equal(covered, vis.astype(np.int32)), (ctx, n, window)


def test_window_start_of_query_block_pair(lib):
    """Query block 1 of a pair starts at most two kv blocks after query block 0
    (the split-KV schedule relies on it)."""
    for ctx in range(0, 700, 7):
        for n in (129, 256, 300, 700):
            for window in (1, 5, 100, 128, 129, 333, 700):
                for qb in range(0, -(-n // 128) - 1):
                    f0 = _lib.first_kv_block(qb, ctx, n, window)
                    f1 = _lib.first_kv_block(qb + 1, ctx, n, window)
                    assert f0 <= f1 <= f0 + 2, (ctx, n, window, qb)


def test_window_validation(lib):
    import ctypes
    P = ctypes.c_void_p(16)
    base = [P, P, P, 1, P, None, 1, 1, 0, 4, 4, 64, 0.125]
    tail = [P, P, 8, P, 8, 16, None, None]
    assert lib.prefill_attn_sliding_window(*base, 0, *tail) == 2     # window < 1
    assert lib.prefill_attn_sliding_window(*base, -3, *tail) == 2
    with_ctx = list(base)
    with_ctx[8] = 5                                                     # max_context_len without context_lens
    assert lib.prefill_attn_sliding_window(*with_ctx, 4, *tail) == 2


def test_decode_validation(lib):
    P = ctypes.c_void_p(FAKE)
    #        q  k  v  ctx B  maxc H  G  D    scale  out cache nb bt mbps bs  status stream
    base = [P, P, P, P, 2, 100, 8, 2, 128, 0.088, P, P, 16, P, 8, 16, None, None]

    def call(**over):
        a = list(base)
        names = ["q", "k", "v", "ctx", "B", "maxc", "H", "G", "D", "scale", "out", "cache", "nb", "bt", "mbps", "bs"]
        for key, val in over.items():
            a[names.index(key)] = val
        return lib.paged_decode_attn(*a)

    assert call(q=None) == 1 and call(ctx=None) == 1 and call(bt=None) == 1
    assert call(H=9, G=2) == 2
    assert call(H=34, G=2) == 3            # 17 query heads per kv head: above 16
    assert call(D=96) == 3 and call(bs=24) == 3 and call(scale=0.0) == 3
    assert call(maxc=128) == 4             # 129 keys do not fit 8 pages of 16
    assert call(nb=0) == 4
    assert call(q=ctypes.c_void_p(FAKE + 4)) == 7
    assert call(B=0) == 0


def test_qkv_projection_validation(lib):
    P = ctypes.c_void_p(FAKE)
    #        x  w  T    hid  H  G  d    q  k  v  status stream
    base = [P, P, 128, 512, 4, 2, 64, P, P, P, None, None]

    def call(**over):
        a = list(base)
        names = ["x", "w", "T", "hid", "H", "G", "d", "q", "k", "v"]
        for key, val in over.items():
            a[names.index(key)] = val
        return lib.qkv_projection(*a)

    assert call(x=None) == 1 and call(v=None) == 1
    assert call(T=-1) == 2 and call(H=0) == 2
    assert call(hid=100) == 3              # hidden not a multiple of 64
    assert call(d=48) == 3                 # head_dim not a multiple of 32
    assert call(H=3, G=1, d=64) == 3       # (3 + 2) * 64 = 320 output features: not a multiple of 256
    assert call(q=ctypes.c_void_p(FAKE + 2)) == 7
    assert call(T=0) == 0


def test_attn_out_projection_validation(lib):
    P = ctypes.c_void_p(FAKE)
    #        o  w  T    H  d    hid  y  status stream
    base = [P, P, 128, 4, 64, 512, P, None, None]

    def call(**over):
        a = list(base)
        names = ["o", "w", "T", "H", "d", "hid", "y"]
        for key, val in over.items():
            a[names.index(key)] = val
        return lib.attn_out_projection(*a)

    assert call(o=None) == 1 and call(y=None) == 1
    assert call(T=-1) == 2 and call(H=0) == 2 and call(hid=0) == 2
    assert call(H=3, d=48) == 3            # 144 input features: not a multiple of 64
    assert call(hid=320) == 3              # hidden not a multiple of 256
    assert call(w=ctypes.c_void_p(FAKE + 2)) == 7
    assert call(T=0) == 0


def test_fp8_entry_points_validation(lib):
    P = ctypes.c_void_p(FAKE)
    #      q  k  v  T    cu B  maxs H  G  D    scale  ks vs out cache nb bt mbps bs status stream
    pre = [P, P, P, 128, P, 1, 128, 4, 2, 128, 0.088, P, P, P, P, 8, P, 8, 16, None, None]
    bad = list(pre); bad[14] = None
    assert lib.prefill_attn_fp8_cache(*bad) == 1         # no FP8 pool
    bad = list(pre); bad[12] = None
    assert lib.prefill_attn_fp8_cache(*bad) == 1         # no V scale
    bad = list(pre); bad[9] = 96
    assert lib.prefill_attn_fp8_cache(*bad) == 3         # head_dim
    bad = list(pre); bad[18] = 24
    assert lib.prefill_attn_fp8_cache(*bad) == 3         # block size
    bad = list(pre); bad[14] = ctypes.c_void_p(FAKE + 4)
    assert lib.prefill_attn_fp8_cache(*bad) == 7         # pool alignment
    bad = list(pre); bad[3] = 0
    assert lib.prefill_attn_fp8_cache(*bad) == 0         # no rows: nothing to do
    #      q  k  v  T   cu ctx B  maxq maxc H  G  D    scale  ks vs out cache nb bt mbps bs status stream
    chk = [P, P, P, 64, P, P, 1, 64, 64, 4, 2, 128, 0.088, P, P, P, P, 8, P, 8, 16, None, None]
    bad = list(chk); bad[5] = None
    assert lib.prefill_attn_chunked_fp8(*bad) == 1       # no context lengths
    bad = list(chk); bad[13] = None
    assert lib.prefill_attn_chunked_fp8(*bad) == 1       # no K scale
    bad = list(chk); bad[9] = 5
    assert lib.prefill_attn_chunked_fp8(*bad) == 2       # 5 query heads over 2 kv heads
    bad = list(chk); bad[11] = 96
    assert lib.prefill_attn_chunked_fp8(*bad) == 3       # head_dim
    bad = list(chk); bad[8] = 129
    assert lib.prefill_attn_chunked_fp8(*bad) == 4       # a 129-token context does not fit 8 pages of 16
    bad = list(chk); bad[16] = ctypes.c_void_p(FAKE + 8)
    assert lib.prefill_attn_chunked_fp8(*bad) == 7       # pool alignment
    bad = list(chk); bad[3] = 0
    assert lib.prefill_attn_chunked_fp8(*bad) == 0       # no rows: nothing to do
    #       k  v  T   cu ctx B  G  D    ks vs cache nb bt mbps bs  status stream
    store = [P, P, 10, P, None, 1, 2, 128, P, P, P, 4, P, 4, 16, None, None]
    # only calls that the host rejects before any launch (the pointers are fake)
    bad = list(store); bad[8] = None
    assert lib.kv_cache_store_fp8(*bad) == 1             # no K scale
    bad = list(store); bad[7] = 96
    assert lib.kv_cache_store_fp8(*bad) == 3             # head_dim
    bad = list(store); bad[14] = 24
    assert lib.kv_cache_store_fp8(*bad) == 3             # block size
    bad = list(store); bad[10] = ctypes.c_void_p(FAKE + 8)
    assert lib.kv_cache_store_fp8(*bad) == 7             # cache alignment
    #      q  k  v  ctx B  maxc H  G  D    scale  ks vs out cache nb bt mbps bs status stream
    dec = [P, P, P, P, 2, 100, 8, 2, 128, 0.088, P, P, P, P, 16, P, 8, 16, None, None]
    bad = list(dec); bad[11] = None
    assert lib.paged_decode_attn_fp8(*bad) == 1          # no V scale
    bad = list(dec); bad[5] = 128
    assert lib.paged_decode_attn_fp8(*bad) == 4          # 129 keys do not fit 8 pages of 16
    bad = list(dec); bad[4] = 0
    assert lib.paged_decode_attn_fp8(*bad) == 0          # nothing to do


def test_header_is_plain_c_and_links_from_c(lib, tmp_path):
    """A C99 program includes the header, links against libprefill.so and calls
    two host-only functions (no device work)."""
    import subprocess
    src = tmp_path / "abi_from_c.c"
    src.write_text(
        '#include <stdio.h>\n#include <string.h>\n#include "prefill.h"\n'
        'int main(void) {\n'
        '    if (strcmp(prefill_status_string(PREFILL_OK), "ok") != 0) return 1;\n'
        '    /* query block 1 of a 300-row prompt with no context: kv blocks 0 and 1 */\n'
        '    if (prefill_num_kv_blocks(1, 0, 300, 128, 128) != 2) return 2;\n'
        '    puts("ok");\n    return 0;\n}\n')
    exe = tmp_path / "abi_from_c"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                           os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lprefill",
                           "-Wl,-rpath," + libdir])
    assert subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.strip() == "ok"


def test_exp2_hook_rejects_bad_arguments(lib):
    lib.prefill_test_exp2_fma2.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    assert lib.prefill_test_exp2_fma2(None, FAKE, 4, None) == 1
    assert lib.prefill_test_exp2_fma2(FAKE, None, 4, None) == 1
    assert lib.prefill_test_exp2_fma2(FAKE, FAKE, -1, None) == 2
