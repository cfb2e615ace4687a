"""Kernel-level parity on the GPU: the tensor-core GEMM and the self-attention kernel
against float64 references of the same (bf16-exact) operands, at sizes that span
several tiles and ragged tails."""
import math

import numpy as np
import pytest

import synth_inputs as si
from oracle import model as om
from gpu_helpers import rel_err, to_dev

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import audio_driven_talking_b200 as fh  # noqa: E402


def _bf16_operands(seed, M, N, K):
    A = si.to_bf16(si.normal(seed, 1, (M, K)).astype(np.float32))
    W = si.to_bf16((si.normal(seed, 2, (N, K)) / math.sqrt(K)).astype(np.float32))
    b = si.normal(seed, 3, (N,)).astype(np.float32)
    return A, W, b


@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (160, 256, 1536), (300, 1536, 256), (1280, 1536, 1536),
                                   (1280, 4608, 1536), (1280, 1536, 8960), (8640, 8960, 1536), (1, 128, 128),
                                   (300, 1536, 1024), (1280, 8960, 1536), (520, 1536, 1536), (4000, 1536, 1536),
                                   (520, 1536, 4096), (4000, 1536, 4096)])
def test_linear_bf16_tensor_core(M, N, K):
    """Single-CTA tiles, and 256-row CTA-pair tiles (cta_group::2) for K >= 1024, N >= 1536."""
    A, W, b = _bf16_operands(M + N + K, M, N, K)
    out = fh.linear(to_dev(A, torch.bfloat16), to_dev(W, torch.bfloat16), to_dev(b))
    torch.cuda.synchronize()
    rows = np.arange(0, M, max(1, M // 512))          # rows are independent: check a sample of them
    ref = A[rows].astype(np.float64) @ W.astype(np.float64).T + b
    # fp32 accumulation of bf16-exact products: error bound ~ K * 2^-24 * sum|a||w|; 1e-3 of RMS is far above it
    assert rel_err(out.cpu().numpy()[rows], ref) < 1e-3


@pytest.mark.parametrize("M,N,K", [(1280, 1536, 1536), (1280, 4608, 1536), (1280, 1536, 8960), (1280, 8960, 1536),
                                   (8640, 8960, 1536), (8640, 1536, 8960), (520, 1536, 1536), (300, 1536, 1024),
                                   (4000, 1536, 4096), (256, 1536, 1024), (864, 4608, 1536)])
def test_linear_bf16_pair_tiles(M, N, K):
    """The CTA-pair GEMMs at the model's projection shapes and ragged row counts: persistent
    pairs with several tiles each, the split-K clusters of four (N = 1536), the last rows of a
    ragged tile; repeated calls agree bitwise."""
    A, W, b = _bf16_operands(M * 3 + N + K, M, N, K)
    Ad, Wd, bd = to_dev(A, torch.bfloat16), to_dev(W, torch.bfloat16), to_dev(b)
    out = fh.linear(Ad, Wd, bd)
    out2 = fh.linear(Ad, Wd, bd)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    rows = np.unique(np.concatenate([np.arange(0, M, max(1, M // 512)), np.arange(max(0, M - 40), M)]))
    ref = A[rows].astype(np.float64) @ W.astype(np.float64).T + b
    assert rel_err(out.cpu().numpy()[rows], ref) < 1e-3


@pytest.mark.parametrize("M,N,K", [(128, 384, 384), (64, 1152, 384), (100, 1024, 384)])
def test_linear_f32_cuda_core(M, N, K):
    A = si.normal(7, 1, (M, K)).astype(np.float32)
    W = (si.normal(7, 2, (N, K)) / math.sqrt(K)).astype(np.float32)
    b = si.normal(7, 3, (N,)).astype(np.float32)
    out = fh.linear(to_dev(A), to_dev(W), to_dev(b))
    torch.cuda.synchronize()
    ref = A.astype(np.float64) @ W.astype(np.float64).T + b
    assert rel_err(out.cpu().numpy(), ref) < 1e-5


def bf16_out_err(gpu, ref) -> float:
    """Error beyond the output's own bf16 rounding (half an ulp, <= 2^-9 |ref|), over RMS(ref)."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    excess = np.maximum(np.abs(g - r) - 2.0 ** -8 * np.abs(r), 0.0)
    return float(np.max(excess) / np.sqrt(np.mean(r * r)))


def _attn_case(seed, B, NH, L, bf16):
    """q, k bf16-exact and v float16-exact values (the types the bf16 model's QKV projection
    stores), or float32 for the fp32 path."""
    q = si.normal(seed, 1, (B, NH, L, 128)).astype(np.float32)
    k = si.normal(seed, 2, (B, NH, L, 128)).astype(np.float32)
    v = si.normal(seed, 3, (B, NH, L, 128)).astype(np.float32)
    if bf16:
        q, k, v = si.to_bf16(q), si.to_bf16(k), v.astype(np.float16).astype(np.float32)
    # per-head partial sums of squares: positive, of the size a unit-RMS row would give
    ssq = (128.0 * (0.5 + si.uniform(seed, 4, (B * L, 2 * NH)))).astype(np.float32)
    return q, k, v, ssq


def _attn_reference(q, k, v, ssq, eps=1e-6):
    B, NH, L, hd = q.shape
    D = NH * hd
    r = 1.0 / np.sqrt(ssq.astype(np.float64).reshape(B, L, 2, NH).sum(-1) / D + eps)  # [B, L, 2]
    qe = q.astype(np.float64).transpose(0, 2, 1, 3) * r[:, :, 0, None, None]
    ke = k.astype(np.float64).transpose(0, 2, 1, 3) * r[:, :, 1, None, None]
    ve = v.astype(np.float64).transpose(0, 2, 1, 3)
    o = om.self_attention(qe, ke, ve, 1.0 / math.sqrt(hd))          # [B, L, NH, hd]
    return o.reshape(B * L, D)


@pytest.mark.parametrize("B,NH,L", [(1, 1, 128), (1, 2, 200), (1, 12, 1280), (2, 3, 2880), (1, 1, 64), (1, 1, 33),
                                   (1, 2, 130)])
def test_attention_bf16_tensor_core(B, NH, L):
    q, k, v, ssq = _attn_case(B * 100 + L, B, NH, L, True)
    out = fh.attention(to_dev(q, torch.bfloat16), to_dev(k, torch.bfloat16), to_dev(v, torch.float16), to_dev(ssq))
    torch.cuda.synchronize()
    ref = _attn_reference(q, k, v, ssq)
    # the weights enter P.V in float16 (11-bit significand, relative step 2^-11), so beyond the
    # bf16 rounding of the stored output there remain their rounding (unbiased, about 2^-12 of
    # each weight; its largest effect over millions of outputs of 2880-key rows is 1.4e-3 of
    # the outputs' RMS), the float32 accumulation and the approximate exponential
    assert bf16_out_err(out.float().cpu().numpy(), ref) < 2e-3


@pytest.mark.parametrize("L", [640, 1280])
def test_attention_bf16_rescales_when_the_row_max_grows(L):
    """Keys whose scale grows along the sequence (x1 to x7) raise every row's maximum score by
    far more than 2^8 from the first key tile to the last, so the kernel's rescaling of its
    accumulators, which it skips while a row's maximum stays within 2^8, runs several times."""
    q, k, v, ssq = _attn_case(7000 + L, 1, 2, L, True)
    ramp = (1.0 + 6.0 * np.arange(L) / L).astype(np.float32)
    k = si.to_bf16(k * ramp[None, None, :, None])
    q = si.to_bf16(q * 2.0)
    out = fh.attention(to_dev(q, torch.bfloat16), to_dev(k, torch.bfloat16), to_dev(v, torch.float16), to_dev(ssq))
    torch.cuda.synchronize()
    ref = _attn_reference(q, k, v, ssq)
    assert bf16_out_err(out.float().cpu().numpy(), ref) < 2e-3


@pytest.mark.parametrize("B,NH,L", [(1, 3, 128), (2, 1, 100)])
def test_attention_f32_cuda_core(B, NH, L):
    q, k, v, ssq = _attn_case(B * 10 + L, B, NH, L, False)
    out = fh.attention(to_dev(q), to_dev(k), to_dev(v), to_dev(ssq))
    torch.cuda.synchronize()
    assert rel_err(out.cpu().numpy(), _attn_reference(q, k, v, ssq)) < 1e-4


def test_attention_rows_sum_to_one_on_gpu():
    """V = ones gives ones for every query (softmax rows sum to 1), ragged key tail included."""
    q, k, _, ssq = _attn_case(5, 1, 2, 300, True)
    v = np.ones_like(q)
    out = fh.attention(to_dev(q, torch.bfloat16), to_dev(k, torch.bfloat16), to_dev(v, torch.float16), to_dev(ssq))
    torch.cuda.synchronize()
    assert np.max(np.abs(out.float().cpu().numpy() - 1.0)) < 1e-2


# ---------------------------------------------------------------------------- cross-attention
def _xattn_case(seed, B, NH, F, HW, bf16):
    D, A = NH * 128, 32
    q = si.normal(seed, 1, (B, F * HW, D)).astype(np.float32)
    kv = si.normal(seed, 2, (B, F, A, 2 * D)).astype(np.float32)
    if bf16:
        q, kv = si.to_bf16(q), si.to_bf16(kv)
    ssq_q = (128.0 * (0.5 + si.uniform(seed, 3, (B * F * HW, NH)))).astype(np.float32)
    ssq_k = (128.0 * (0.5 + si.uniform(seed, 4, (B * F * A, NH)))).astype(np.float32)
    return q, kv, ssq_q, ssq_k


def _xattn_reference(q, kv, ssq_q, ssq_k, F, eps=1e-6):
    """oracle.model.frame_cross_attention on the RMS-scaled queries and keys (reading R4)."""
    B, L, D = q.shape
    NH, A = D // 128, kv.shape[2]
    rq = 1.0 / np.sqrt(ssq_q.astype(np.float64).reshape(B, L, NH).sum(-1) / D + eps)
    rk = 1.0 / np.sqrt(ssq_k.astype(np.float64).reshape(B, F, A, NH).sum(-1) / D + eps)
    qe = (q.astype(np.float64) * rq[..., None]).reshape(B, L, NH, 128)
    ke = (kv[..., :D].astype(np.float64) * rk[..., None]).reshape(B, F, A, NH, 128)
    ve = kv[..., D:].astype(np.float64).reshape(B, F, A, NH, 128)
    return om.frame_cross_attention(qe, ke, ve, F, 1.0 / math.sqrt(128)).reshape(B, L, D)


def _xattn(q, kv, ssq_q, ssq_k, F, dt=None):
    dt = dt or torch.bfloat16
    out = fh.cross_attention(to_dev(q, dt), to_dev(ssq_q), to_dev(kv, dt), to_dev(ssq_k), F)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("B,NH,F,HW", [(1, 12, 5, 256), (1, 12, 5, 576), (2, 3, 3, 144), (1, 2, 2, 100)])
def test_cross_attention_bf16_tensor_core(B, NH, F, HW):
    """1280 and 2880 tokens of the model's shapes, and frames that end inside a 128-query tile
    (12 x 12 and 100 tokens per frame): rows past a frame are neither read nor written."""
    q, kv, sq, sk = _xattn_case(B * 1000 + HW, B, NH, F, HW, True)
    got = _xattn(q, kv, sq, sk, F)
    assert bf16_out_err(got, _xattn_reference(q, kv, sq, sk, F)) < 1e-3


@pytest.mark.parametrize("B,NH,F,HW", [(1, 3, 2, 64), (2, 1, 3, 50)])
def test_cross_attention_f32_cuda_core(B, NH, F, HW):
    q, kv, sq, sk = _xattn_case(B * 10 + HW, B, NH, F, HW, False)
    got = _xattn(q, kv, sq, sk, F, torch.float32)
    assert rel_err(got, _xattn_reference(q, kv, sq, sk, F)) < 1e-4


def test_cross_attention_frame_locality_on_gpu():
    """Changing frame 1's audio keys and values changes the rows of frame 1 only; every other
    row is bitwise the same."""
    B, NH, F, HW = 1, 12, 5, 256
    q, kv, sq, sk = _xattn_case(31, B, NH, F, HW, True)
    a = _xattn(q, kv, sq, sk, F)
    kv2 = kv.copy()
    kv2[:, 1] = si.to_bf16(kv2[:, 1] * 1.5 + 0.25)
    b = _xattn(q, kv2, sq, sk, F)
    frame = np.arange(F * HW) // HW
    assert np.array_equal(a[:, frame != 1], b[:, frame != 1])
    assert np.max(np.abs(a[:, frame == 1] - b[:, frame == 1])) > 1e-2


def test_cross_attention_identical_keys_return_the_value_on_gpu():
    """With the 32 audio tokens of a frame all equal (one distinct key and value) every
    softmax weight is 1/32 and each output row is that value, exactly."""
    B, NH, F, HW = 1, 3, 2, 144
    q, kv, sq, sk = _xattn_case(32, B, NH, F, HW, True)
    kv[:, :, :] = kv[:, :, :1]
    sk = sk.reshape(B, F, 32, NH)
    sk[:, :, :] = sk[:, :, :1]
    sk = sk.reshape(B * F * 32, NH)
    got = _xattn(q, kv, sq, sk, F)
    want = np.repeat(kv[:, :, 0, NH * 128:], HW, axis=1)
    assert np.array_equal(got, want)


def test_cross_attention_is_invariant_to_the_order_of_a_frames_audio_tokens():
    """Permuting a frame's 32 audio tokens (keys, values and their sums of squares together)
    leaves the output unchanged up to the order of the fp32 sums: at most one step of the
    stored bf16 value (2^-7 of it) where that order moves a rounding boundary."""
    B, NH, F, HW = 1, 4, 3, 160
    q, kv, sq, sk = _xattn_case(33, B, NH, F, HW, True)
    a = _xattn(q, kv, sq, sk, F)
    perm = np.array(si.normal(34, 1, (32,))).argsort()
    kv2 = kv[:, :, perm]
    sk2 = sk.reshape(B, F, 32, NH)[:, :, perm].reshape(B * F * 32, NH)
    b = _xattn(q, kv2, sq, sk2, F)
    assert np.max(np.abs(a - b) - 2.0 ** -7 * np.abs(a)) <= 1e-6
    assert np.mean(a != b) < 0.05
