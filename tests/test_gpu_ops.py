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
    q = si.normal(seed, 1, (B, NH, L, 128)).astype(np.float32)
    k = si.normal(seed, 2, (B, NH, L, 128)).astype(np.float32)
    v = si.normal(seed, 3, (B, NH, L, 128)).astype(np.float32)
    if bf16:
        q, k, v = si.to_bf16(q), si.to_bf16(k), si.to_bf16(v)
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
    out = fh.attention(to_dev(q, torch.bfloat16), to_dev(k, torch.bfloat16), to_dev(v, torch.bfloat16), to_dev(ssq))
    torch.cuda.synchronize()
    ref = _attn_reference(q, k, v, ssq)
    # the weights enter P.V as two bf16 parts (about 16 bits), so beyond the bf16 rounding of the
    # stored output only the float32 accumulation and the approximate exponential remain
    assert bf16_out_err(out.float().cpu().numpy(), ref) < 1e-3


@pytest.mark.parametrize("L", [640, 1280])
def test_attention_bf16_rescales_when_the_row_max_grows(L):
    """Keys whose scale grows along the sequence (x1 to x7) raise every row's maximum score by
    far more than 2^8 from the first key tile to the last, so the kernel's rescaling of its
    accumulators, which it skips while a row's maximum stays within 2^8, runs several times."""
    q, k, v, ssq = _attn_case(7000 + L, 1, 2, L, True)
    ramp = (1.0 + 6.0 * np.arange(L) / L).astype(np.float32)
    k = si.to_bf16(k * ramp[None, None, :, None])
    q = si.to_bf16(q * 2.0)
    out = fh.attention(to_dev(q, torch.bfloat16), to_dev(k, torch.bfloat16), to_dev(v, torch.bfloat16), to_dev(ssq))
    torch.cuda.synchronize()
    ref = _attn_reference(q, k, v, ssq)
    assert bf16_out_err(out.float().cpu().numpy(), ref) < 1e-3


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
    out = fh.attention(to_dev(q, torch.bfloat16), to_dev(k, torch.bfloat16), to_dev(v, torch.bfloat16), to_dev(ssq))
    torch.cuda.synchronize()
    assert np.max(np.abs(out.float().cpu().numpy() - 1.0)) < 1e-2
