"""Pins for the CPU oracle: each check ties it to something other than itself -- a figure
the pages print, a hand-derived layout example, a closed form, an invariant, a library
routine (numpy / torch) on a special case, or brute force on tiny inputs.

Every check is a ``pin_*`` function taking an oracle instance, so that
``test_oracle_mutants.py`` can run the same checks against deliberately broken copies
of the oracle (built on the CPU) and show that each plausible mistake fails one of them.
"""

import json
import math
import os

import numpy as np
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
B, T, T3 = oracle.BINARY, oracle.TERNARY, oracle.TERNARY_B3


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _exact_x(M, K, seed):
    """x with small dyadic values (multiples of 1/8 in [-4, 4]); products with fp16 scales
    that are powers of two and all partial sums are exact in fp64, so any summation order
    gives the same bits."""
    rng = np.random.default_rng(seed)
    return (rng.integers(-32, 33, size=(M, K)) / 8.0).astype(np.float16)


def _pow2_scales(N, G, seed):
    rng = np.random.default_rng(seed)
    return (2.0 ** rng.integers(-6, 3, size=(N, G))).astype(np.float16)


# --------------------------------------------------------------------------------------
# Number formats (library routines: numpy float16, torch bfloat16)
# --------------------------------------------------------------------------------------

def pin_f16_decode(o):
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([o.f16_value(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def pin_bf16_decode(o):
    bits = torch.arange(0, 65536, 7, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([o.bf16_value(int(b) & 0xFFFF) for b in bits.tolist()])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])


def pin_bf16_round(o):
    rng = np.random.default_rng(1)
    # fp32-exact inputs so torch's float->bf16 conversion rounds once (ties to even)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),          # bf16 subnormals
        np.array([1.00390625, 1.01171875, -1.00390625, 3.0e38, -3.4e38, 0.0], np.float32),
    ]).astype(np.float64)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = o.to_bf16_bits(v)
    assert np.array_equal(got, ref)


def pin_f16_round(o):
    rng = np.random.default_rng(2)
    v = np.concatenate([
        rng.standard_normal(5000) * 100.0,
        rng.standard_normal(2000) * 1e-6,                                  # fp16 subnormals
        np.array([65504.0, 65519.0, 65520.0, -70000.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]),
    ])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    got = o.to_f16_bits(v)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------------------------
# Layout: hand-derived examples
# --------------------------------------------------------------------------------------

def pin_layout_examples(o):
    g = _golden("layout_examples.json")
    for ex in g["binary"]:
        K = ex["K"]
        q = -np.ones((1, K), np.int8)
        q[0, ex["plus_one_at"]] = 1
        st, words, _ = o.pack(B, q, np.ones((1, K // 128), np.float16))
        assert st == oracle.OK
        assert [f"{w:08x}" for w in words[0]] == ex["words_hex"]
        back, bad = o.unpack(B, words, K)
        assert bad == 0 and np.array_equal(back, q)
    for ex in g["ternary"]:
        K = ex["K"]
        q = np.full((1, K), ex["default"], np.int8)
        for k, v in ex["values_at"].items():
            q[0, int(k)] = v
        st, words, _ = o.pack(T, q, np.ones((1, K // 128), np.float16))
        assert st == oracle.OK
        assert [f"{w:08x}" for w in words[0]] == ex["words_hex"]
        back, bad = o.unpack(T, words, K)
        assert bad == 0 and np.array_equal(back, q)


def pin_scale_index(o):
    """Weight (n, k) takes the scale of row n, group k // 128."""
    N, K = 3, 384
    s = np.array([[1, 2, 4], [8, 16, 32], [0.5, 0.25, 0.125]], np.float16)
    q = np.ones((N, K), np.int8)
    _, words, s_out = o.pack(B, q, s)
    W = o.dequant(B, words, s_out, K)
    for n in range(N):
        for k in (0, 127, 128, 255, 256, 383):
            assert W[n, k] == float(s[n, k // 128])


# --------------------------------------------------------------------------------------
# Round trips
# --------------------------------------------------------------------------------------

def pin_roundtrip_binary(o):
    N, K = 7, 640
    words = synth.binary_words(3, N, K).numpy().view(np.uint32)
    q, bad = o.unpack(B, words, K)
    assert bad == 0 and set(np.unique(q)) <= {-1, 1}
    st, words2, _ = o.pack(B, q, np.ones((N, K // 128), np.float16))
    assert st == oracle.OK and np.array_equal(words2, words)


def pin_roundtrip_ternary(o):
    N, K = 5, 512
    q = synth.random_ternary(4, synth.TID_TERNARY, (N, K)).numpy()
    st, words, _ = o.pack(T, q, np.ones((N, K // 128), np.float16))
    assert st == oracle.OK
    back, bad = o.unpack(T, words, K)
    assert bad == 0 and np.array_equal(back, q)
    st, words2, _ = o.pack(T, back, np.ones((N, K // 128), np.float16))
    assert np.array_equal(words2, words)


def pin_invalid_codes(o):
    K = 128
    for fmt, badv in ((B, 0), (B, 2), (B, -2), (T, 2), (T, -2)):
        q = np.ones((1, K), np.int8) if fmt == B else np.zeros((1, K), np.int8)
        q[0, 77] = badv
        st, _, _ = o.pack(fmt, q, np.ones((1, 1), np.float16))
        assert st == oracle.ERR_CODE
    # ternary code 3 in a packed word is reported by unpack
    words = np.zeros((1, 8), np.uint32)
    words[0, 2] = 0x3 << 6                       # field 3 of word 2 = k = 35
    q, bad = o.unpack(T, words, K)
    assert bad == 1 and q[0, 35] == 0
    assert np.isnan(o.dequant(T, words, np.ones((1, 1), np.float16), K)[0, 35])
    assert o.words_per_row(B, 100) == -1 and o.words_per_row(T, 0) == -1


# --------------------------------------------------------------------------------------
# Base-3 ternary storage
# --------------------------------------------------------------------------------------

def pin_b3_examples(o):
    """Hand-derived bytes (tests/golden/b3_examples.json) for the base-3 layout."""
    for ex in _golden("b3_examples.json")["cases"]:
        K = ex["K"]
        q = np.full((1, K), ex["default"], np.int8)
        for k, v in ex["values_at"].items():
            q[0, int(k)] = v
        st, b, _ = o.pack(T3, q, np.ones((1, K // 128), np.float16))
        assert st == oracle.OK and b.shape == (1, 26 * K // 128)
        if "all_bytes" in ex:
            expect = np.array(ex["all_bytes"], np.uint8)
        else:
            expect = np.zeros(26 * K // 128, np.uint8)
            for off, v in ex["nonzero_bytes"].items():
                expect[int(off)] = v
        assert np.array_equal(b[0], expect), ex["why"]
        back, bad = o.unpack(T3, b, K)
        assert bad == 0 and np.array_equal(back, q)


def pin_b3_byte_values(o):
    """Every one of the 256 byte values at every byte position: exactly 3^5 = 243 values
    decode as five codes and 3^4 = 81 as four (each v written once), and a valid byte's
    codes are the base-3 digits of floor(byte * 3^n / 256), first digit most significant."""
    K = 128
    rows = np.repeat(np.arange(256, dtype=np.uint8)[:, None], 26, axis=1)
    q, _ = o.unpack(T3, rows, K)
    valid5, valid4 = set(), set()
    for byte in range(256):
        _, bad = o.unpack(T3, rows[byte:byte + 1], K)
        assert bad in (0, 2, 24, 26)
        if bad in (0, 2):
            valid5.add(byte)
            v = byte * 243 // 256
            digits = [(v // 3 ** (4 - p)) % 3 - 1 for p in range(5)]
            assert list(q[byte, :5]) == digits and list(q[byte, 115:120]) == digits
        if bad in (0, 24):
            valid4.add(byte)
            v = byte * 81 // 256
            digits = [(v // 3 ** (3 - p)) % 3 - 1 for p in range(4)]
            assert list(q[byte, 120:124]) == digits and list(q[byte, 124:128]) == digits
    assert len(valid5) == 243 and len(valid4) == 81
    assert sorted(valid5) == sorted({-(-256 * v // 243) for v in range(243)})
    assert sorted(valid4) == sorted({-(-256 * v // 81) for v in range(81)})
    # an invalid byte: its codes unpack as 0 and its weights are NaN
    bad_byte = min(set(range(256)) - valid5)
    one = np.zeros((1, 26), np.uint8)
    one[0, 3] = bad_byte
    qq, bad = o.unpack(T3, one, K)
    assert bad == 1 and np.all(qq[0, 15:20] == 0)
    w = o.dequant(T3, one, np.ones((1, 1), np.float16), K)
    assert np.all(np.isnan(w[0, 15:20])) and not np.any(np.isnan(w[0, :15]))


def pin_b3_equals_2bit(o):
    """Base-3 storage holds the same ternary weights as the (separately pinned) 2-bit
    storage: dequant, GEMV (fp64, k ascending, so bit for bit) and embedding agree; the
    round trip gives back the codes, over ragged block counts."""
    for N, K, M in ((5, 128, 2), (4, 1024, 1), (3, 1280, 3), (2, 2176, 8)):
        q = synth.random_ternary(19, 2, (N, K)).numpy()
        s = synth.scales(19, N, K // 128).numpy()
        st3, b3, s3 = o.pack(T3, q, s)
        st2, w2, s2 = o.pack(T, q, s)
        assert st3 == st2 == oracle.OK and np.array_equal(s3, s2)
        back, bad = o.unpack(T3, b3, K)
        assert bad == 0 and np.array_equal(back, q)
        assert np.array_equal(o.dequant(T3, b3, s3, K), o.dequant(T, w2, s2, K))
        assert np.array_equal(o.dequant(T3, b3, s3, K), _dense(q, s))
        xb = synth.activations(20, M, K, dtype=torch.bfloat16)
        y3, b_3 = o.gemv(T3, xb, oracle.X_BF16, b3, s3, K)
        y2, b_2 = o.gemv(T, xb, oracle.X_BF16, w2, s2, K)
        assert np.array_equal(y3, y2) and np.array_equal(b_3, b_2)
        ids = np.array([N - 1, 0, N, -3], np.int32)
        e3, bad3 = o.embed(T3, ids, b3, s3, K)
        e2, bad2 = o.embed(T, ids, w2, s2, K)
        assert bad3 == bad2 == 2 and np.array_equal(e3, e2)
    for badv in (2, -2, 5):
        q = np.zeros((1, 256), np.int8)
        q[0, 200] = badv
        assert o.pack(T3, q, np.ones((1, 2), np.float16))[0] == oracle.ERR_CODE
    assert o.row_bytes(T3, 128) == 26 and o.row_bytes(T3, 5120) == 1040 and o.row_bytes(T3, 100) == -1


def pin_b3_bits_per_weight(o):
    """Stored size from the oracle's buffers: 26 bytes + one fp16 scale per 128 weights is
    1.75 bits per weight, between the pages' 1.71 (log2 3 + 16/128) and the 2.125 of the
    2-bit storage."""
    g = _golden("pages_figures.json")
    bpw3 = _stored_bpw(o, T3, K=1152)
    assert bpw3 == 1.75
    assert g["ternary_true_bits_per_weight"]["value"] < bpw3 < _stored_bpw(o, T)
    assert math.log2(3) + 16 / 128 < bpw3


# --------------------------------------------------------------------------------------
# SwiGLU MLP (model card "Model overview")
# --------------------------------------------------------------------------------------

def _mlp_case(o, seed, M, K, F, N, fmt_gu=None):
    fmt_gu = T if fmt_gu is None else fmt_gu
    rng = np.random.default_rng(seed)
    qg = synth.random_ternary(seed, 2, (F, K)).numpy() if fmt_gu == T else synth.random_signs(seed, 1, (F, K)).numpy()
    qu = synth.random_ternary(seed, 3, (F, K)).numpy() if fmt_gu == T else synth.random_signs(seed, 4, (F, K)).numpy()
    qd = synth.random_signs(seed, 5, (N, F)).numpy()
    sg = (2.0 ** rng.integers(-4, 0, size=(F, K // 128))).astype(np.float16)
    su = (2.0 ** rng.integers(-4, 0, size=(F, K // 128))).astype(np.float16)
    sd = (2.0 ** rng.integers(-6, -2, size=(N, F // 128))).astype(np.float16)
    x = _exact_x(M, K, seed + 1)
    packs = [o.pack(fmt_gu, qg, sg), o.pack(fmt_gu, qu, su), o.pack(B, qd, sd)]
    assert all(p[0] == oracle.OK for p in packs)
    return x, (qg, sg), (qu, su), (qd, sd), [(p[1], p[2]) for p in packs]


def pin_mlp_vs_numpy(o):
    """Dense numpy fp64: W = q * s for the three matrices, g, u, a = g sigma(g) u, y = a Wd^T."""
    for fmt_gu in (T, B):
        x, g_, u_, d_, packed = _mlp_case(o, 41, 3, 256, 256, 200, fmt_gu)
        a, y, b = o.mlp_swiglu(x, oracle.X_F16, fmt_gu, packed[0], packed[1], B, packed[2])
        xs = x.astype(np.float64)
        g = xs @ _dense(*g_).T
        u = xs @ _dense(*u_).T
        a_ref = g * (1.0 / (1.0 + np.exp(-g))) * u
        assert np.allclose(a, a_ref, rtol=1e-12, atol=1e-300)
        y_ref = a_ref @ _dense(*d_).T
        assert np.allclose(y, y_ref, rtol=1e-9, atol=1e-12 * np.max(np.abs(y_ref)))
        b_ref = 2e-3 * (np.abs(a_ref) @ np.abs(_dense(*d_)).T)
        assert np.allclose(b, b_ref, rtol=1e-9)


def pin_mlp_silu_identities(o):
    """silu(z) - silu(-z) = z; silu(z) ~ z for large z and ~ 0 for large -z; zero up codes give
    a = 0 and y = 0."""
    K, F, N = 128, 128, 128
    x = np.zeros((1, K), np.float16)
    x[0, 0] = 1.0
    qg = np.ones((F, K), np.int8)
    qg[1::2] = -1                                    # gate row 2i+1 = -(gate row 2i)
    sg = np.full((F, 1), 2.0, np.float16)
    sg[4:6] = 32768.0                                # g = +-32768 for rows 4, 5
    qu = np.ones((F, K), np.int8)                   # u = s_u = 1
    su = np.ones((F, 1), np.float16)
    qd = np.ones((N, F), np.int8)
    sd = np.ones((N, 1), np.float16)
    pg, pu, pd = o.pack(T, qg, sg), o.pack(T, qu, su), o.pack(B, qd, sd)
    a, y, b = o.mlp_swiglu(x, oracle.X_F16, T, pg[1:], pu[1:], B, pd[1:])
    for i in (0, 2, 6):
        g = float(sg[i, 0])
        assert abs((a[0, i] - a[0, i + 1]) - g) <= 1e-15 * g
    assert abs(a[0, 4] - 32768.0) <= 1e-9 and abs(a[0, 5]) <= 1e-300
    qz = np.zeros((F, K), np.int8)
    pz = o.pack(T, qz, su)
    a0, y0, _ = o.mlp_swiglu(x, oracle.X_F16, T, pg[1:], pz[1:], B, pd[1:])
    assert np.all(a0 == 0) and np.all(y0 == 0)


# --------------------------------------------------------------------------------------
# Dense -> g128 quantiser (least-squares fit per group; the pages do not give the method)
# --------------------------------------------------------------------------------------

def _f16(v):
    return np.float16(v).view(np.uint16)            # numpy rounds fp64 to fp16 to nearest even


def pin_quantize_hand(o):
    w = np.zeros((3, 128), np.float32)
    w[0, :3] = [3, -3, 1]                           # scores 9, 36/2, 49/3: support {0, 1}, s = 3
    w[1, ::2], w[1, 1::2] = 2, -2
    # row 2: all zeros
    qt, st = o.quantize(T, w)
    assert qt[0, :3].tolist() == [1, -1, 0] and np.all(qt[0, 3:] == 0) and st[0, 0] == _f16(3.0)
    assert np.all(qt[1] == np.where(w[1] > 0, 1, -1)) and st[1, 0] == _f16(2.0)
    assert np.all(qt[2] == 0) and st[2, 0] == _f16(0.0)
    qb, sb = o.quantize(B, w)
    assert np.all(qb == np.where(w >= 0, 1, -1))
    assert sb[0, 0] == _f16(7 / 128) and sb[1, 0] == _f16(2.0) and sb[2, 0] == _f16(0.0)


def pin_quantize_score_tie(o):
    """An exact tie of the score (sum of the j largest |w|)^2 / j between two supports: |w| =
    3, 1, 1, 1 gives 9 at j = 1 and 36 / 4 = 9 at j = 4 (8 and 25/3 between), all exact in
    binary64; the smaller support is taken, so s = 3 rather than 1.5."""
    w = np.zeros((2, 128), np.float32)
    w[0, :4] = [3, -1, 1, -1]
    w[1, [5, 40, 77, 120]] = [-1, 1, -3, 1]              # the same magnitudes elsewhere in a group
    q, s = o.quantize(T, w)
    assert q[0, :4].tolist() == [1, 0, 0, 0] and np.all(q[0, 4:] == 0) and s[0, 0] == _f16(3.0)
    expect = np.zeros(128, np.int8)
    expect[77] = -1
    assert np.array_equal(q[1], expect) and s[1, 0] == _f16(3.0)


def pin_quantize_binary_closed_form(o):
    rng = np.random.default_rng(31)
    w = (rng.normal(size=(6, 640)) * 0.02).astype(np.float32)
    q, s = o.quantize(B, w)
    assert np.array_equal(q, np.where(w >= 0, 1, -1).astype(np.int8))
    mean = np.abs(w.astype(np.float64)).reshape(6, 5, 128).mean(axis=2)
    assert np.array_equal(s, _f16(mean))


def pin_quantize_ternary_bruteforce(o):
    """Groups with at most 10 non-zero weights: the oracle's support is the subset of them with
    the smallest squared error, found by trying all 2^10 subsets."""
    import itertools
    rng = np.random.default_rng(32)
    for trial in range(40):
        w = np.zeros((1, 128), np.float32)
        nz = rng.choice(128, size=int(rng.integers(1, 11)), replace=False)
        w[0, nz] = (rng.normal(size=len(nz)) * rng.uniform(0.1, 3)).astype(np.float32)
        q, s = o.quantize(T, w)
        a = np.abs(w[0, nz].astype(np.float64))
        tot = float(np.sum(w[0].astype(np.float64) ** 2))
        best, best_set = tot, ()
        for r in range(1, len(nz) + 1):
            for sub in itertools.combinations(range(len(nz)), r):
                err = tot - float(np.sum(a[list(sub)])) ** 2 / r
                if err < best - 1e-12:
                    best, best_set = err, sub
        support = sorted(int(nz[i]) for i in best_set)
        assert sorted(np.nonzero(q[0])[0].tolist()) == support
        assert np.all(q[0, support] == np.sign(w[0, support]))
        mean = np.mean(a[list(best_set)]) if best_set else 0.0
        assert s[0, 0] == _f16(mean)


def pin_quantize_invariants(o):
    rng = np.random.default_rng(33)
    w = (rng.normal(size=(4, 256)) * 0.05).astype(np.float32)
    w[w == 0] = 1e-3
    for fmt in (B, T):
        q, s = o.quantize(fmt, w)
        q4, s4 = o.quantize(fmt, 4 * w)
        assert np.array_equal(q4, q)
        assert np.array_equal(s4.view(np.float16).astype(np.float64), 4 * s.view(np.float16).astype(np.float64))
        qn, sn = o.quantize(fmt, -w)
        assert np.array_equal(qn, -q) and np.array_equal(sn, s)


# --------------------------------------------------------------------------------------
# Top-k and sampling (model card "Generation parameters": temperature 0.7, top-p 0.95, top-k 20)
# --------------------------------------------------------------------------------------

def pin_topk_hand(o):
    idx, vals = o.topk(np.array([[1.0, 5.0, 3.0, 5.0, -2.0], [0.0, 0.0, 0.0, -1.0, 2.0]]), 3)
    assert idx.tolist() == [[1, 3, 2], [4, 0, 1]]
    assert vals.tolist() == [[5.0, 5.0, 3.0], [2.0, 0.0, 0.0]]


def pin_topk_vs_numpy(o):
    """Against numpy's lexsort (value descending, then index ascending), with many ties."""
    rng = np.random.default_rng(21)
    for N, k in ((1000, 20), (37, 37), (5000, 1), (300, 32)):
        y = np.round(rng.normal(size=(3, N)) * 4) / 4          # a few hundred distinct values
        idx, vals = o.topk(y, k)
        for m in range(3):
            order = np.lexsort((np.arange(N), -y[m]))[:k]
            assert idx[m].tolist() == order.tolist()
            assert vals[m].tolist() == y[m, order].tolist()


def pin_sample_hand(o):
    """Hand-worked probabilities: logits with exact exponentials."""
    ln2 = math.log(2.0)
    v2, i2 = np.array([0.0, 0.0]), np.array([7, 9])
    assert o.sample_topk(v2, i2, 1.0, 1.0, 0.49) == 7 and o.sample_topk(v2, i2, 1.0, 1.0, 0.51) == 9
    # top-p 0.5: the first candidate alone reaches it
    assert o.sample_topk(v2, i2, 1.0, 0.5, 0.9) == 7
    # p proportional to 4, 2, 1: cumulative 4/7, 6/7; top-p 0.8 keeps two, renormalised 2/3, 1/3
    v3, i3 = np.array([2 * ln2, ln2, 0.0]), np.array([30, 10, 20])
    assert o.sample_topk(v3, i3, 1.0, 0.8, 0.62) == 30
    assert o.sample_topk(v3, i3, 1.0, 0.8, 0.70) == 10
    assert o.sample_topk(v3, i3, 1.0, 1.0, 0.80) == 10 and o.sample_topk(v3, i3, 1.0, 1.0, 0.90) == 20
    # temperature 0.5 squares the ratios: 16, 4, 1 -> cumulative 16/21, 20/21
    assert o.sample_topk(v3, i3, 0.5, 1.0, 0.75) == 30 and o.sample_topk(v3, i3, 0.5, 1.0, 0.77) == 10
    assert o.sample_topk(v3, i3, 0.5, 1.0, 0.96) == 20


def pin_sample_frequencies(o):
    """Over a fine grid of u the draws follow softmax(v / T) restricted to the top-p prefix."""
    rng = np.random.default_rng(22)
    v = np.sort(rng.normal(size=20))[::-1] * 3
    ids = np.arange(100, 120)
    T, top_p = 0.7, 0.95
    p = np.exp((v - v[0]) / T)
    p /= p.sum()
    keep = int(np.searchsorted(np.cumsum(p), top_p) + 1)
    q = p[:keep] / p[:keep].sum()
    us = (np.arange(20000) + 0.5) / 20000
    draws = np.array([o.sample_topk(v, ids, T, top_p, u) for u in us])
    assert set(np.unique(draws)) <= set(ids[:keep].tolist())
    freq = np.array([np.mean(draws == ids[i]) for i in range(keep)])
    assert np.max(np.abs(freq - q)) <= 1.5 / 20000


# --------------------------------------------------------------------------------------
# Mapping and closed forms
# --------------------------------------------------------------------------------------

def pin_mapping_closed_form(o):
    """All-ones group -> s * sum(x); all-zeros -> -s * sum(x)."""
    K = 256
    x = _exact_x(2, K, 5)
    s = np.array([[0.5, 4.0], [0.5, 4.0]], np.float16)
    words = np.zeros((2, K // 32), np.uint32)
    words[0, :] = 0xFFFFFFFF                     # row 0: every bit 1
    y, _ = o.gemv(B, x, oracle.X_F16, words, s, K)
    xs = x.astype(np.float64)
    for m in range(2):
        expect1 = 0.5 * math.fsum(xs[m, :128]) + 4.0 * math.fsum(xs[m, 128:])
        assert y[m, 0] == expect1
        assert y[m, 1] == -expect1


def pin_bound_closed_form(o):
    K = 128
    x = np.array([[1.0, -2.0] + [0.0] * 126], np.float16)
    words = np.zeros((1, 4), np.uint32)
    _, b = o.gemv(B, x, oracle.X_F16, words, np.array([[0.25]], np.float16), K)
    assert b[0, 0] == 2e-3 * (0.25 + 0.5)
    tw = np.full((1, 8), 0x55555555, np.uint32)   # ternary all-zero codes: scale still counts
    _, bt = o.gemv(T, x, oracle.X_F16, tw, np.array([[0.25]], np.float16), K)
    assert bt[0, 0] == 2e-3 * (0.25 + 0.5)


# --------------------------------------------------------------------------------------
# Brute force: dense fp64 matmul (numpy) of W = q * s built directly from the inputs
# --------------------------------------------------------------------------------------

def _dense(q, s):
    return q.astype(np.float64) * np.repeat(s.astype(np.float64), 128, axis=1)


def pin_bruteforce_exact(o):
    for fmt, N, K, M in ((B, 9, 256, 3), (T, 6, 384, 8), (B, 1, 128, 1)):
        q = (synth.random_signs(6, 1, (N, K)) if fmt == B
             else synth.random_ternary(6, 2, (N, K))).numpy()
        s = _pow2_scales(N, K // 128, 7)
        x = _exact_x(M, K, 8)
        st, words, s_out = o.pack(fmt, q, s)
        assert st == oracle.OK
        y, _ = o.gemv(fmt, x, oracle.X_F16, words, s_out, K)
        ref = x.astype(np.float64) @ _dense(q, s).T
        assert np.array_equal(y, ref)


def pin_bruteforce_random(o):
    N, K, M = 33, 512, 4
    q = synth.random_signs(9, 1, (N, K)).numpy()
    s = synth.scales(9, N, K // 128).numpy()
    xb = synth.activations(9, M, K, dtype=torch.bfloat16)
    st, words, s_out = o.pack(B, q, s)
    y, b = o.gemv(B, xb, oracle.X_BF16, words, s_out, K)
    ref = xb.to(torch.float64).numpy() @ _dense(q, s).T
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
    # the bound by brute force: 2e-3 * |x| @ |W|^T
    bref = 2e-3 * (np.abs(xb.to(torch.float64).numpy()) @ np.abs(_dense(q, s)).T)
    assert np.allclose(b, bref, rtol=1e-12, atol=0)


def pin_dequant_vs_dense(o):
    N, K = 4, 256
    for fmt in (B, T):
        q = (synth.random_signs(10, 1, (N, K)) if fmt == B
             else synth.random_ternary(10, 2, (N, K))).numpy()
        s = synth.scales(10, N, K // 128).numpy()
        _, words, s_out = o.pack(fmt, q, s)
        assert np.array_equal(o.dequant(fmt, words, s_out, K), _dense(q, s))


# --------------------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------------------

def pin_invariants(o):
    N, K, M = 5, 256, 2
    x = _exact_x(M, K, 11)
    s = _pow2_scales(N, K // 128, 12)
    words = synth.binary_words(13, N, K).numpy().view(np.uint32)
    y, _ = o.gemv(B, x, oracle.X_F16, words, s, K)
    # flipping every bit negates y
    yn, _ = o.gemv(B, x, oracle.X_F16, ~words, s, K)
    assert np.array_equal(yn, -y)
    # scaling every scale by 2^j scales y by 2^j
    y4, _ = o.gemv(B, x, oracle.X_F16, words, (s.astype(np.float64) * 4).astype(np.float16), K)
    assert np.array_equal(y4, 4 * y)
    # ternary with codes in {0, 2} equals binary with bit = code / 2
    q, _ = o.unpack(B, words, K)
    _, tw, _ = o.pack(T, q, s)
    yt, _ = o.gemv(T, x, oracle.X_F16, tw, s, K)
    assert np.array_equal(yt, y)
    # ternary with every code 1 (value 0) gives exactly 0
    z, _ = o.gemv(T, x, oracle.X_F16, np.full((N, K // 16), 0x55555555, np.uint32), s, K)
    assert np.all(z == 0.0)
    # linearity in x (exact values)
    x2 = _exact_x(M, K, 14)
    ya, _ = o.gemv(B, x2, oracle.X_F16, words, s, K)
    yab, _ = o.gemv(B, (x.astype(np.float64) + x2.astype(np.float64)).astype(np.float16),
                    oracle.X_F16, words, s, K)
    assert np.array_equal(yab, y + ya)


def pin_bf16_x(o):
    """bf16 and fp16 encodings of the same values give the same y."""
    K = 128
    x16 = _exact_x(1, K, 15)
    xbf = torch.from_numpy(x16.astype(np.float32)).to(torch.bfloat16)
    words = synth.binary_words(16, 3, K).numpy().view(np.uint32)
    s = _pow2_scales(3, 1, 17)
    y1, _ = o.gemv(B, x16, oracle.X_F16, words, s, K)
    y2, _ = o.gemv(B, xbf, oracle.X_BF16, words, s, K)
    assert np.array_equal(y1, y2)


# --------------------------------------------------------------------------------------
# Embedding
# --------------------------------------------------------------------------------------

def pin_embed(o):
    N, K = 50, 256
    q = synth.random_signs(18, 1, (N, K)).numpy()
    s = synth.scales(18, N, K // 128).numpy()
    _, words, s_out = o.pack(B, q, s)
    ids = np.array([3, 0, 49, 3, 17], np.int32)
    out, bad = o.embed(B, ids, words, s_out, K)
    assert bad == 0 and np.array_equal(out, _dense(q, s)[ids])
    # bf16 rounding of the gathered rows equals torch's (fp16 values are fp32-exact)
    ref = torch.from_numpy(out.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.to_bf16_bits(out), ref)
    out2, bad2 = o.embed(B, np.array([-1, 50, 2], np.int32), words, s_out, K)
    assert bad2 == 2 and np.all(out2[:2] == 0) and np.array_equal(out2[2], _dense(q, s)[2])


# --------------------------------------------------------------------------------------
# Sizes and the pages' printed figures
# --------------------------------------------------------------------------------------

def _stored_bpw(o, fmt, N=4, K=1280):
    """Stored bits per weight from the sizes of the oracle's packed buffers."""
    q = np.ones((N, K), np.int8)
    st, words, s_out = o.pack(fmt, q, np.ones((N, K // 128), np.float16))
    assert st == oracle.OK
    return (words.nbytes + s_out.nbytes) * 8 / (N * K)


def pin_bits_per_weight(o):
    g = _golden("pages_figures.json")
    bpw_b = _stored_bpw(o, B)
    bpw_t = _stored_bpw(o, T)
    assert bpw_b == g["bits_per_weight_binary"]["value"]
    assert bpw_t == 2.125                           # 2-bit codes + the same 16-bit scale per 128
    assert round(g["fp16_bits_per_weight"]["value"] / bpw_b, 1) == g["reduction_vs_fp16"]["value"]
    # MLX scale+bias form: two fp16 values per group
    mlx = (1 + 2 * 16 / 128)
    assert mlx == g["mlx_bits_per_weight"]["value"]
    P = g["language_params_billion"]["value"] * 1e9
    assert abs(P * bpw_b / 8 / 1e9 - g["binary_deploy_gb"]["value"]) <= g["binary_deploy_gb"]["tol"]
    assert abs(P * 16 / 8 / 1e9 - g["fp16_gb"]["value"]) <= g["fp16_gb"]["tol"]
    assert abs(P * bpw_t / 8 / 1e9 - g["ternary_deploy_gb_2bit_storage"]["value"]) <= \
        g["ternary_deploy_gb_2bit_storage"]["tol"]
    true_t = math.log2(3) + 16 / 128
    assert round(true_t, 2) == g["ternary_true_bits_per_weight"]["value"]
    assert abs(P * true_t / 8 / 1e9 - g["ternary_theoretical_gb"]["value"]) <= g["ternary_theoretical_gb"]["tol"]
    assert round(bpw_t / bpw_b, 1) == g["ternary_over_binary_bytes_per_step"]["value"]
    # untied embedding + LM head: 2 * vocab * hidden ~ 2.5B
    eh = 2 * g["vocab_size"]["value"] * g["hidden_size"]["value"] / 1e9
    assert round(eh, 1) == g["embed_lmhead_params_billion"]["value"]
    assert g["hidden_size"]["value"] % g["group_size"]["value"] == 0


def pin_mlx_identity(o):
    """s_mlx = 2 s, bias = -s reproduces +-s bit-exactly for every finite non-zero fp16 s
    with |2s| finite (for s = +-0 the sum s + (-s) is +0, equal in value)."""
    checked = 0
    for sb in range(65536):
        s = o.f16_value(sb)
        if not math.isfinite(s) or abs(2 * s) > 65504:
            continue
        if s == 0.0:
            assert o.f16_value(o.mlx_affine_dequant(sb, 0)) == 0.0
            assert o.f16_value(o.mlx_affine_dequant(sb, 1)) == 0.0
            continue
        assert o.mlx_affine_dequant(sb, 1) == sb
        assert o.mlx_affine_dequant(sb, 0) == sb ^ 0x8000
        checked += 1
    assert checked > 60000


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


def test_f16_decode(orc): pin_f16_decode(orc)
def test_bf16_decode(orc): pin_bf16_decode(orc)
def test_bf16_round(orc): pin_bf16_round(orc)
def test_f16_round(orc): pin_f16_round(orc)
def test_layout_examples(orc): pin_layout_examples(orc)
def test_scale_index(orc): pin_scale_index(orc)
def test_roundtrip_binary(orc): pin_roundtrip_binary(orc)
def test_roundtrip_ternary(orc): pin_roundtrip_ternary(orc)
def test_invalid_codes(orc): pin_invalid_codes(orc)
def test_mapping_closed_form(orc): pin_mapping_closed_form(orc)
def test_bound_closed_form(orc): pin_bound_closed_form(orc)
def test_bruteforce_exact(orc): pin_bruteforce_exact(orc)
def test_bruteforce_random(orc): pin_bruteforce_random(orc)
def test_dequant_vs_dense(orc): pin_dequant_vs_dense(orc)
def test_invariants(orc): pin_invariants(orc)
def test_bf16_x(orc): pin_bf16_x(orc)
def test_embed(orc): pin_embed(orc)
def test_bits_per_weight(orc): pin_bits_per_weight(orc)
def test_mlx_identity(orc): pin_mlx_identity(orc)
def test_b3_examples(orc): pin_b3_examples(orc)
def test_b3_byte_values(orc): pin_b3_byte_values(orc)
def test_b3_equals_2bit(orc): pin_b3_equals_2bit(orc)
def test_b3_bits_per_weight(orc): pin_b3_bits_per_weight(orc)
def test_mlp_vs_numpy(orc): pin_mlp_vs_numpy(orc)
def test_mlp_silu_identities(orc): pin_mlp_silu_identities(orc)
def test_quantize_hand(orc): pin_quantize_hand(orc)
def test_quantize_score_tie(orc): pin_quantize_score_tie(orc)
def test_quantize_binary_closed_form(orc): pin_quantize_binary_closed_form(orc)
def test_quantize_ternary_bruteforce(orc): pin_quantize_ternary_bruteforce(orc)
def test_quantize_invariants(orc): pin_quantize_invariants(orc)
def test_topk_hand(orc): pin_topk_hand(orc)
def test_topk_vs_numpy(orc): pin_topk_vs_numpy(orc)
def test_sample_hand(orc): pin_sample_hand(orc)
def test_sample_frequencies(orc): pin_sample_frequencies(orc)
