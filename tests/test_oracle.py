"""Pins for the CPU oracle (no GPU).

The oracle is only trusted once it is tied to something other than itself:
hand-worked values (tests/golden/hand_cases.json), the IEEE binary16 format as
numpy implements it, textbook integer and fp64 matrix products (numpy
matmul), the quantize/dequantize round-trip bound, code-range invariants, and
an independent numpy restatement that must agree bit for bit.

Readings of the Atom pages pinned here: 128-element groups quantized
independently and a 128-channel high-precision outlier group ("Atom
(mixed-precision block-outlier low-bit quantization for serving)", fields
"Weight group size" and "notes"); INT4 bulk plus higher-precision outlier
channels (same page, "Activation scheme").
"""
import json
import os

import numpy as np
import pytest

from w4a4_mixed_precision_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _idx(spec: str):
    return np.array(eval(spec, {"range": range}), dtype=np.int32)  # noqa: S307 (fixture literal)


def _fill(spec, n):
    v = np.full(n, spec.get("fill", 0), dtype=np.float64)
    head = spec.get("head", [])
    v[:len(head)] = head
    return v


def _hex_bytes(spec: str, n: int, tail_fill: int = 0):
    if "x" in spec:
        h, count = spec.split("x")
        return np.full(int(count), int(h, 16), dtype=np.uint8)
    out = np.full(n, tail_fill, dtype=np.uint8)
    b = bytes.fromhex(spec)
    out[:len(b)] = np.frombuffer(b, dtype=np.uint8)
    return out


def _f32_div(num, den):
    return np.float32(num) / np.float32(den)   # one correctly rounded fp32 division


# --------------------------------------------------------------------------- fp16 format


def test_f16_decode_matches_ieee_binary16_for_every_pattern(c_oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([c_oracle.f16_to_f32(int(b)) for b in bits], dtype=np.float32)
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    assert (got[~nan].view(np.uint32) == ref[~nan].view(np.uint32)).all()


def test_f32_to_f16_rounds_to_nearest_even(c_oracle):
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.standard_normal(2000) * 300, [2049.0, 2051.0, 1.0 + 2 ** -11,
                                                            65504.0, 1e-8, -3.0000001]])
    vals = vals.astype(np.float32)
    ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([c_oracle.f32_to_f16(float(v)) for v in vals], dtype=np.uint16)
    assert (got == ref).all()


# --------------------------------------------------------------------------- hand-worked


def _check_quant_fixture(quantize_fn):
    """Run every hand-worked quantize case through quantize_fn; return a list of failures."""
    g = _golden()
    bad = []
    for case in g["quantize"]:
        K = case["K"]
        idx = _idx(case["outlier_idx"])
        perm_dense = np.setdiff1d(np.arange(K), idx)
        if case["name"].startswith("identity"):
            for r, row in enumerate(case["rows"]):
                x = np.zeros(K)
                x[perm_dense] = _fill(row["x_dense"], K - 128)
                x[idx] = _fill(row["x_outlier"], 128)
                q4, q8, sc = quantize_fn(x.astype(np.float16)[None, :], idx)
                want4 = _hex_bytes(row["q4_hex"], 64, row.get("q4_tail_fill", 0))
                want8 = _fill(row["q8"], 128).astype(np.int8)
                wants = np.array([_f32_div(*p) for p in row["scales"]], dtype=np.float32)
                if not (q4[0] == want4).all():
                    bad.append((case["name"], r, "q4"))
                if not (q8[0] == want8).all():
                    bad.append((case["name"], r, "q8"))
                if not (sc[:, 0].view(np.uint32) == wants.view(np.uint32)).all():
                    bad.append((case["name"], r, "scales"))
        else:
            x = np.zeros(K)
            j = np.arange(128)
            x[2 * j] = (j % 15) - 7
            x[2 * j + 1] = j - 64
            q4, q8, sc = quantize_fn(x.astype(np.float16)[None, :], idx)
            if not (q4[0, :8] == _hex_bytes(case["q4_head_hex"], 8)).all():
                bad.append((case["name"], "q4 head"))
            # every dense code equals its value because the dense scale is exactly 1
            lo = (q4[0] & 0xF).astype(int)
            hi = (q4[0] >> 4).astype(int)
            nib = np.empty(128, dtype=int)
            nib[0::2], nib[1::2] = lo, hi
            nib = np.where(nib >= 8, nib - 16, nib)
            if not (nib == (j % 15) - 7).all():
                bad.append((case["name"], "dense codes"))
            for t, v in case["q8_at"].items():
                if int(q8[0, int(t)]) != v:
                    bad.append((case["name"], "q8", t))
            wants = np.array([_f32_div(*p) for p in case["scales"]], dtype=np.float32)
            if not (sc[:, 0].view(np.uint32) == wants.view(np.uint32)).all():
                bad.append((case["name"], "scales"))
    return bad


def test_hand_quantize_cases_c(c_oracle):
    assert _check_quant_fixture(c_oracle.quantize) == []


def test_hand_quantize_cases_numpy(np_oracle):
    assert _check_quant_fixture(np_oracle.quantize) == []


def _hand_gemm_operands():
    g = _golden()["gemm"]
    K = g["K"]

    def row(spec):
        dense = np.full(K - 128, spec.get("dense_fill", 0), dtype=np.float64)
        if "dense_alternate_from_1" in spec:
            a, b = spec["dense_alternate_from_1"]
            dense[1::2] = a
            dense[2::2] = b
        dense[:len(spec["dense_head"])] = spec["dense_head"]
        out = np.full(128, spec.get("outlier_fill", 0), dtype=np.float64)
        out[:len(spec["outlier_head"])] = spec["outlier_head"]
        return np.concatenate([dense, out])

    A = np.stack([row(s) for s in g["A"]]).astype(np.float16)
    W = np.stack([row(s) for s in g["W"]]).astype(np.float16)
    return g, K, _idx(g["outlier_idx"]), A, W


def test_hand_gemm_partials_and_output(c_oracle, np_oracle):
    g, K, idx, A, W = _hand_gemm_operands()
    qa = c_oracle.quantize(A, idx)
    qw = c_oracle.quantize(W, idx)
    assert (qa[2] == 1.0).all() and (qw[2] == 1.0).all()
    P = c_oracle.partials(qa[0], qa[1], qw[0], qw[1], K)
    assert P.tolist() == g["P"]
    Y = c_oracle.gemm(*qa, *qw, K)
    assert Y.tolist() == [[float(v) for v in r] for r in g["Y"]]
    assert np_oracle.partials(qa[0], qa[1], qw[0], qw[1]).tolist() == g["P"]


# --------------------------------------------------------------------------- structure


@pytest.mark.parametrize("K,seed", [(256, 1), (512, 2), (4096, 3), (11008, 4)])
def test_permutation_structure(c_oracle, K, seed):
    rng = np.random.default_rng(seed)
    idx = rng.choice(K, 128, replace=False).astype(np.int32)     # unsorted on purpose
    perm = c_oracle.permutation(K, idx)
    assert sorted(perm.tolist()) == list(range(K))                # a bijection
    dense = perm[:K - 128]
    assert (np.diff(dense) > 0).all()                             # ascending
    assert set(dense.tolist()).isdisjoint(idx.tolist())
    assert (perm[K - 128:] == idx).all()                          # tail in list order


@pytest.mark.parametrize("bad", ["dup", "neg", "big"])
def test_oracle_rejects_bad_outlier_lists(c_oracle, np_oracle, bad):
    idx = np.arange(128, dtype=np.int32)
    if bad == "dup":
        idx[5] = idx[6]
    elif bad == "neg":
        idx[0] = -1
    else:
        idx[0] = 256
    x = np.zeros((1, 256), dtype=np.float16)
    with pytest.raises(c_oracle.OracleError):
        c_oracle.quantize(x, idx)
    with pytest.raises(ValueError):
        np_oracle.quantize(x, idx)


# --------------------------------------------------------------------------- invariants


def _cases():
    A0, W0, i0 = inputs.activations(0), inputs.weights(0), inputs.outlier_channels(0)
    yield "tiny", A0, W0, i0
    A1, W1, i1 = inputs.activations(1, rows=8), inputs.weights(1, rows=48), inputs.outlier_channels(1)
    yield "decode_slice", A1, W1, i1
    A2, W2, i2 = inputs.random_case(11, 37, 45, 640, dist="t", param=3.0, outlier_factor=50.0,
                                    sorted_outliers=False)
    yield "ragged_unsorted", A2, W2, i2


CASES = list(_cases())


@pytest.mark.parametrize("name,A,W,idx", CASES, ids=[c[0] for c in CASES])
def test_roundtrip_bound_and_code_range(c_oracle, name, A, W, idx):
    K = A.shape[1]
    perm = c_oracle.permutation(K, idx)
    for X in (A, W):
        q4, q8, sc = c_oracle.quantize(X, idx)
        dq = c_oracle.dequantize(q4, q8, sc, K)
        xr = X.astype(np.float64)[:, perm]
        s = np.repeat(sc.T.astype(np.float64), 128, axis=1)
        # |x - q*scale| <= scale/2 * (1 + 6*qmax*u), u = 2^-24: scale, inv and
        # t = x*inv are each rounded once in fp32 and |t| <= qmax (derivation in
        # the design notes); 7*qmax*u leaves room for the second-order terms.
        qm = np.where(np.arange(K) < K - 128, 7.0, 127.0)[None, :]
        assert (np.abs(xr - dq) <= s / 2 * (1 + 7 * qm * 2.0 ** -24)).all()
        lo, hi = (q4 & 0xF).astype(int), (q4 >> 4).astype(int)
        nibs = np.concatenate([lo, hi], axis=1)
        nibs = np.where(nibs >= 8, nibs - 16, nibs)
        assert nibs.min() >= -7 and nibs.max() <= 7
        assert q8.min() >= -127
        # the element at the group amax maps to +-qmax
        G = K // 128
        xg = np.abs(xr).reshape(X.shape[0], G, 128)
        dqg = np.abs(dq).reshape(X.shape[0], G, 128)
        arg = xg.argmax(axis=2)
        top = np.take_along_axis(dqg, arg[:, :, None], axis=2)[:, :, 0]
        qmax = np.array([7.0] * (G - 1) + [127.0])
        nz = sc.T > 0
        ratio = top / np.where(nz, sc.T, 1)
        assert np.allclose(ratio[nz], np.broadcast_to(qmax, ratio.shape)[nz])


@pytest.mark.parametrize("name,A,W,idx", CASES, ids=[c[0] for c in CASES])
def test_output_equals_fp64_product_of_dequantized_operands(c_oracle, name, A, W, idx):
    K = A.shape[1]
    qa = c_oracle.quantize(A, idx)
    qw = c_oracle.quantize(W, idx)
    Y = c_oracle.gemm(*qa, *qw, K)
    ref = c_oracle.dequantize(*qa, K) @ c_oracle.dequantize(*qw, K).T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


@pytest.mark.parametrize("name,A,W,idx", CASES, ids=[c[0] for c in CASES])
def test_numpy_restatement_agrees_bit_for_bit(c_oracle, np_oracle, name, A, W, idx):
    K = A.shape[1]
    qa_c, qw_c = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    qa_n, qw_n = np_oracle.quantize(A, idx), np_oracle.quantize(W, idx)
    for a, b in zip(qa_c + qw_c, qa_n + qw_n):
        assert a.shape == b.shape
        assert (a.view(np.uint8) == b.view(np.uint8)).all()
    P_c = c_oracle.partials(qa_c[0], qa_c[1], qw_c[0], qw_c[1], K)
    P_n = np_oracle.partials(qa_n[0], qa_n[1], qw_n[0], qw_n[1])
    assert (P_c == P_n).all()
    Y = c_oracle.gemm(*qa_c, *qw_c, K)
    assert np.allclose(Y, np_oracle.output64(P_n, qa_n[2], qw_n[2]), rtol=1e-13, atol=1e-300)


def test_lossless_integer_inputs_give_the_textbook_integer_matmul(c_oracle):
    """T4: integer inputs whose every group has amax exactly qmax quantize with
    scale 1 and codes equal to the inputs, so Y is the plain integer matmul of
    the permuted operands."""
    rng = np.random.default_rng(99)
    M, N, K = 9, 13, 640
    idx = rng.choice(K, 128, replace=False).astype(np.int32)
    perm = c_oracle.permutation(K, idx)

    def make(rows):
        xr = np.zeros((rows, K))
        xr[:, :K - 128] = rng.integers(-7, 8, (rows, K - 128))
        xr[:, K - 128:] = rng.integers(-127, 128, (rows, 128))
        G = K // 128
        for g in range(G):                         # force amax == qmax in every group
            qmax = 7 if g < G - 1 else 127
            col = g * 128 + rng.integers(0, 128, rows)
            xr[np.arange(rows), col] = qmax * rng.choice([-1, 1], rows)
        x = np.zeros_like(xr)
        x[:, perm] = xr                            # place reordered values at source channels
        return x, xr

    A, Ar = make(M)
    W, Wr = make(N)
    qa = c_oracle.quantize(A.astype(np.float16), idx)
    qw = c_oracle.quantize(W.astype(np.float16), idx)
    assert (qa[2] == 1).all() and (qw[2] == 1).all()
    Y = c_oracle.gemm(*qa, *qw, K)
    ref = Ar.astype(np.int64) @ Wr.astype(np.int64).T
    assert (Y == ref).all()
    # the reorder does not change the unquantized product
    assert (A.astype(np.int64) @ W.astype(np.int64).T == ref).all()


def test_partials_sum_to_the_integer_matmul_per_group(c_oracle):
    A, W, idx = inputs.random_case(5, 6, 7, 512)
    K = 512
    qa, qw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    P = c_oracle.partials(qa[0], qa[1], qw[0], qw[1], K)
    from oracle import numpy_oracle as no
    ca, cw = no.codes(qa[0], qa[1]), no.codes(qw[0], qw[1])
    for g in range(K // 128):
        assert (P[g] == ca[:, g * 128:(g + 1) * 128] @ cw[:, g * 128:(g + 1) * 128].T).all()


# --------------------------------------------------------------------------- planted mistakes


@pytest.mark.parametrize("mistake", ["truncate", "half_up", "nibbles_swapped", "scale_by_8",
                                     "no_reorder"])
def test_pins_catch_planted_mistakes(np_oracle, mistake):
    """Each plausible slip in the encoding, planted in a copy of the numpy oracle,
    must fail at least one hand-worked pin."""
    def buggy(x, idx):
        opts = {}
        if mistake == "truncate":
            opts["rounding"] = np.trunc
        elif mistake == "half_up":
            opts["rounding"] = lambda t: np.floor(t + 0.5)
        elif mistake == "nibbles_swapped":
            opts["high_nibble_first"] = True
        elif mistake == "scale_by_8":
            opts["int4_qmax"] = 8.0
        elif mistake == "no_reorder":
            opts["reorder"] = False
        return np_oracle.quantize(x, idx, **opts)
    assert _check_quant_fixture(buggy) != []
