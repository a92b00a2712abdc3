"""GPU check of the error bound the quantizer's certificate assumes for its
tensor-core scores ([TS] Metodologia 3: nearest codeword of one global codebook;
the codes must be the exact nearest codewords, so every decision the tensor
scores make alone has to be covered by a bound).

The certificate takes a tensor score to lie within (tensor_bound in quantize.cu)
    (2^-16 (||a|| max||c|| + max||c||^2 / 2) + ||a|| max||c - fp16(c)||
     + 2^-25 sqrt(8) (max||c|| + ||a||)) * 1.01 + 1.2e-7
of the exact score a . c - ||c||^2 / 2 (cosine rule: a . c_hat, bias 0).  The
2^-16 term is an assumption about the MMA (its accumulation order and rounding
are the hardware's); the others are exact: the fp16 operand of a codebook that is
not fp16-representable, and fp16 lo parts of a (or of c_hat) that fall below the
normal range.  Here the raw accumulators of the same staging, operand build and
MMAs (nsn_selftest_tensor_scores) are compared with fp64 arithmetic over
sub-vector rows of every scale, down to rows whose lo parts are subnormal, for the
fixture codebooks (fp16 values), a codebook that is not fp16-representable and the
cosine rule.  Against the score with the operands the MMA is given (fp16(c) in
place of c) the error must stay within half of the bound's MMA and subnormal
part; against the exact score within the whole bound (its fp16-operand part is
Cauchy-Schwarz and can be nearly tight).  The error against the bare per-pair
2^-16 (sum |a_i c_i| + |bias|) term is printed as well.
"""
import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn
import nsn_testlib as tl

pytestmark = pytest.mark.gpu
TC_REL = 2.0 ** -16


def tensor_scores(rows: np.ndarray, cb: np.ndarray, assign: int) -> np.ndarray:
    r = torch.from_numpy(rows.astype(np.float32)).cuda()
    c = torch.from_numpy(cb.astype(np.float32)).cuda()
    out = torch.full((rows.shape[0], 256), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nsn.nsn_selftest_tensor_scores(r, c, assign, out, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.cpu().numpy().astype(np.float64)


def kernel_bound(rows: np.ndarray, cb32: np.ndarray, assign: int):
    """The certificate's bound per row, from the codebook maxima stage_codebook forms, as
    (its MMA and subnormal part, its fp16-operand part ||a|| max||c - fp16(c)||)."""
    c = cb32.astype(np.float64)
    if assign == 1:
        nrm = np.sqrt((c * c).sum(axis=1, keepdims=True))
        c = np.where(nrm > 0, (c / np.where(nrm > 0, nrm, 1.0)).astype(np.float32), 0.0).astype(np.float64)
        cdel = 0.0
    else:
        e = ((c - c.astype(np.float16).astype(np.float64)) ** 2).sum(axis=1).max()
        cdel = np.sqrt(e) * 1.001 if e > 0 else 0.0
    cmax2 = (c * c).sum(axis=1).max() * 1.0001
    cmax = np.sqrt(cmax2) * 1.0001
    na = np.linalg.norm(rows.astype(np.float32).astype(np.float64), axis=1) * 1.0001
    subn = 2.0 ** -25 * 2.8285
    mma = (TC_REL * (1.001 * na * cmax + 0.5 * cmax2) + subn * (cmax + na)) * 1.01 + 1.2e-7
    return mma, na * cdel * 1.01


def exact_and_terms(rows: np.ndarray, cb32: np.ndarray, assign: int):
    """(exact score, score with the operands the MMA is given, bare 2^-16 term per row and codeword)."""
    a = rows.astype(np.float32).astype(np.float64)
    c = cb32.astype(np.float64)
    if assign == 1:  # unit codewords as the kernel forms them: fp64 norm and division, rounded to fp32
        nrm = np.sqrt((c * c).sum(axis=1, keepdims=True))
        c = np.where(nrm > 0, (c / np.where(nrm > 0, nrm, 1.0)).astype(np.float32), 0.0).astype(np.float64)
        hi = c.astype(np.float16).astype(np.float64)
        c_op = hi + (c - hi).astype(np.float16).astype(np.float64)  # B operands: c_hat_hi, then c_hat_lo
        bias = np.zeros(c.shape[0])
    else:
        c_op = c.astype(np.float16).astype(np.float64)
        bias = -0.5 * (c * c).sum(axis=1)
    exact = a @ c.T + bias[None, :]
    model = a @ c_op.T + bias[None, :]
    return exact, model, TC_REL * (np.abs(a) @ np.abs(c).T + np.abs(bias)[None, :])


def row_sets(rs: np.random.RandomState, abs_mode: bool):
    # sub-vectors of u (unit-variance entries), their tails, tiny and large scales
    for scale in (1.0, 3.0, 0.02, 40.0, 1e-3, 1e-4):
        x = rs.normal(size=(128, 8)) * scale
        yield np.abs(x) if abs_mode else x
    x = rs.normal(size=(128, 8))
    x[:, :4] *= 1e-4  # half of the dims far below the rest
    yield np.abs(x) if abs_mode else x
    x = np.zeros((128, 8))
    x[:, rs.randint(0, 8)] = rs.normal(size=128) * 5.0  # one dominant dimension
    yield np.abs(x) if abs_mode else x


@pytest.mark.parametrize("mode,assign,kind", [(1, 0, "fixture"), (2, 0, "fixture"), (1, 0, "fp32"),
                                              (1, 1, "fixture"), (2, 1, "fixture")])
def test_tensor_scores_within_the_assumed_bound(mode, assign, kind):
    rs = np.random.RandomState(100 + 10 * mode + assign)
    cb = tl.codebook(mode).astype(np.float32)
    if kind == "fp32":  # not fp16-representable: the operand is its fp16 rounding
        cb = (cb + rs.normal(size=cb.shape).astype(np.float32) * 1e-3).astype(np.float32)
        assert np.abs(cb.astype(np.float16).astype(np.float32) - cb).max() > 0
    worst_mma, worst_all, worst_term = 0.0, 0.0, 0.0
    for rows in row_sets(rs, mode == 2):
        got = tensor_scores(rows, cb, assign)
        exact, model, term = exact_and_terms(rows, cb, assign)
        mma, fp16_part = kernel_bound(rows, cb, assign)
        assert np.isfinite(got).all()
        worst_mma = max(worst_mma, float((np.abs(got - model) / mma[:, None]).max()))
        worst_all = max(worst_all, float((np.abs(got - exact) / (mma + fp16_part)[:, None]).max()))
        worst_term = max(worst_term, float((np.abs(got - model) / term).max()))
    print(f"mode {mode} assign {assign} {kind}: MMA error up to {worst_mma:.4f} of its part of the bound "
          f"({worst_term:.3g} of the bare per-pair 2^-16 term); total error up to {worst_all:.4f} of the bound")
    assert worst_mma < 0.5, f"MMA error reaches {worst_mma:.3f} of its part of the certificate's bound"
    assert worst_all < 1.0, f"tensor-score error reaches {worst_all:.3f} of the certificate's bound"


def test_selftest_rejects_invalid_arguments():
    r = torch.zeros((129, 8), dtype=torch.float32, device="cuda")
    c = torch.zeros((256, 8), dtype=torch.float32, device="cuda")
    out = torch.zeros((129, 256), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(nsn.NsnError):
        nsn.nsn_selftest_tensor_scores(r, c, 0, out, status)  # more than 128 rows
    with pytest.raises(nsn.NsnError):
        nsn.nsn_selftest_tensor_scores(r[:4], c, 2, out[:4], status)  # unknown rule
