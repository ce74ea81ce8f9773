"""Single-kernel parity against fp64 definitions, through the C ABI (GPU).

Expected values are the plain definitions in float64 on the same bf16/fp32
inputs: the projection y = x W^T, and causal GQA attention from the oracle.
Tolerances follow from the arithmetic (fp32 accumulation; bf16 rounding of the
softmax weights and of the output), stated per test.
"""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _rand(shape, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(dtype)


def _proj_check(x, W, y_gpu, rel=2e-5):
    """|y - x W^T| <= rel * (|x| |W|^T) + 1e-6: fp32 accumulation of K bf16 products."""
    x64, w64 = O.f64(x), O.f64(W)
    ref = x64 @ w64.T
    bound = rel * (np.abs(x64) @ np.abs(w64).T) + 1e-6
    err = np.abs(O.f64(y_gpu) - ref)
    assert np.all(err <= bound), f"max err {err.max():.3e}, worst ratio {(err / bound).max():.2f}"


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (100, 512, 128), (128, 256, 4096), (300, 768, 1024),
                                   (2048, 1024, 4096), (129, 256, 14336)])
def test_gemm_tcgen05_matches_definition(lib, M, N, K):
    import llama_decoder_forward_fwd_b200 as L
    A = _rand((M, K), torch.bfloat16, 1).to(DEV)
    B = _rand((N, K), torch.bfloat16, 2, 0.02).to(DEV)
    C = torch.full((M, N), float("nan"), device=DEV)
    L.llm_op_gemm_bf16(A, B, C)
    torch.cuda.synchronize()
    _proj_check(A.cpu(), B.cpu(), C.cpu())


@pytest.mark.parametrize("M,N,K", [(1, 16, 64), (1, 4096, 4096), (3, 100, 200), (8, 1024, 14336),
                                   (9, 64, 1024), (16, 4096, 4096), (1, 32000, 4096),
                                   # 65 k blocks per row, ~3.5 units per CTA: staged k ranges wrap
                                   # past a row's end and stop short of K
                                   (16, 1000, 4136)])
def test_gemv_matches_definition(lib, M, N, K):
    import llama_decoder_forward_fwd_b200 as L
    x = _rand((M, K), torch.bfloat16, 3).to(DEV)
    W = _rand((N, K), torch.bfloat16, 4, 0.02).to(DEV)
    y = torch.full((M, N), float("nan"), device=DEV)
    ws = torch.full((L.llm_op_gemv_workspace(N, K),), 255, dtype=torch.uint8, device=DEV)
    for _ in range(2):  # the second call reuses the workspace the first left behind
        L.llm_op_gemv_bf16(x, W, y, ws)
    torch.cuda.synchronize()
    _proj_check(x.cpu(), W.cpu(), y.cpu())


def _attn_case(B, T, H, Hk, d, S_max, pos0, dtype, seed):
    q = _rand((B, T, H, d), dtype, seed)
    kc = _rand((B, Hk, S_max, d), dtype, seed + 1)
    vc = _rand((B, Hk, S_max, d), dtype, seed + 2)
    ref = np.empty((B, T, H * d))
    for b in range(B):
        n = pos0[b] + T
        qp = pos0[b] + np.arange(T)
        k = O.f64(kc[b, :, :n, :]).transpose(1, 0, 2)
        v = O.f64(vc[b, :, :n, :]).transpose(1, 0, 2)
        ref[b] = O.attention(O.f64(q[b]), k, v, qp, np.arange(n))
    return q, kc, vc, ref


ATTN_CASES = [
    # B, T, H, Hk, pos0
    (1, 1, 32, 8, [0]),
    (2, 7, 8, 2, [0, 5]),
    (2, 130, 8, 2, [0, 64]),
    (1, 300, 32, 8, [0]),
    (2, 64, 4, 4, [3, 0]),
    (1, 20, 32, 1, [0]),       # multi-query: 32 query heads share one KV head
    (2, 9, 24, 1, [3, 0]),
    (1, 400, 8, 2, [100]),     # four 128-key tiles, a prompt continuing a cache
]


@pytest.mark.parametrize("B,T,H,Hk,pos0", ATTN_CASES)
def test_flash_attention_prefill_matches_oracle(lib, B, T, H, Hk, pos0):
    import llama_decoder_forward_fwd_b200 as L
    d, S = 128, 512
    q, kc, vc, ref = _attn_case(B, T, H, Hk, d, S, pos0, torch.bfloat16, 11)
    out = torch.full((B, T, H * d), float("nan"), dtype=torch.bfloat16, device=DEV)
    p = torch.tensor(pos0, dtype=torch.int32, device=DEV)
    L.llm_op_attention_prefill(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out)
    torch.cuda.synchronize()
    # softmax weights and the output are rounded to bf16: |err| <= 3 * 2^-9 * max|v|.
    err = np.abs(O.f64(out.cpu()) - ref)
    assert err.max() <= 8e-3 * float(vc.abs().max()), err.max()


def test_flash_attention_prefill_rescales_when_scores_grow(lib):
    """Later keys score far higher than earlier ones (key norms growing along the
    cache), so a row's running maximum grows by more than 2^8 between key tiles
    and the accumulated output is rescaled in tensor memory."""
    import llama_decoder_forward_fwd_b200 as L
    B, T, H, Hk, d, S, pos0 = 1, 384, 8, 2, 128, 512, [0]
    g = torch.Generator().manual_seed(21)
    q = (torch.randn(B, T, H, d, generator=g) * 0.5).to(torch.bfloat16)
    grow = (1.0 + torch.arange(S, dtype=torch.float32) / 16.0).view(1, 1, S, 1)
    kc = (torch.randn(B, Hk, S, d, generator=g) * grow).to(torch.bfloat16)
    vc = torch.randn(B, Hk, S, d, generator=g).to(torch.bfloat16)
    ref = np.empty((B, T, H * d))
    k = O.f64(kc[0, :, :T, :]).transpose(1, 0, 2)
    v = O.f64(vc[0, :, :T, :]).transpose(1, 0, 2)
    ref[0] = O.attention(O.f64(q[0]), k, v, np.arange(T), np.arange(T))
    # the scores do grow by more than 2^8 (log2 domain) from the first key tile to the last
    qf, kf = O.f64(q[0, :, 0]), O.f64(kc[0, 0, :T])
    sc = qf @ kf.T / np.sqrt(d) * np.log2(np.e)
    assert (sc[T - 1, 256:T].max() - sc[T - 1, :128].max()) > 8
    out = torch.full((B, T, H * d), float("nan"), dtype=torch.bfloat16, device=DEV)
    p = torch.tensor(pos0, dtype=torch.int32, device=DEV)
    L.llm_op_attention_prefill(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out)
    torch.cuda.synchronize()
    err = np.abs(O.f64(out.cpu()) - ref)
    assert err.max() <= 8e-3 * float(vc.abs().max()), err.max()


@pytest.mark.parametrize("dtype,d,tol", [(torch.bfloat16, 128, 6e-3), (torch.float32, 48, 2e-5),
                                         (torch.float32, 128, 2e-5)])
@pytest.mark.parametrize("B,T,H,Hk,pos0", [(1, 1, 32, 8, [0]), (3, 1, 32, 8, [0, 37, 700]),
                                           (2, 4, 8, 2, [9, 0]), (1, 8, 6, 6, [0]), (2, 3, 12, 3, [100, 1]),
                                           # multi-query (G = 32, 24): a work item takes 16 of a
                                           # token's query heads; with G = 24 chunks straddle tokens
                                           (1, 1, 32, 1, [500]), (2, 3, 32, 1, [100, 7]), (1, 2, 24, 1, [50])])
def test_split_kv_attention_matches_oracle(lib, dtype, d, tol, B, T, H, Hk, pos0):
    import llama_decoder_forward_fwd_b200 as L
    S = 1024
    q, kc, vc, ref = _attn_case(B, T, H, Hk, d, S, pos0, dtype, 21)
    out = torch.full((B, T, H * d), float("nan"), dtype=dtype, device=DEV)
    p = torch.tensor(pos0, dtype=torch.int32, device=DEV)
    ws = torch.empty(L.llm_op_attention_decode_workspace(B, T, H, Hk, d), dtype=torch.uint8, device=DEV)
    for _ in range(2):  # the second call reuses the workspace the first left behind
        L.llm_op_attention_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out, ws)
    torch.cuda.synchronize()
    err = np.abs(O.f64(out.cpu()) - ref)
    assert err.max() <= tol * float(vc.abs().max()), err.max()


@pytest.mark.parametrize("B,H,Hk,S,pos0", [
    (1, 32, 8, 2304, [2048]),          # the benchmark's decode: 8 groups, 8 CTAs per cluster
    (1, 32, 8, 2304, [0]),             # a single key
    (1, 32, 8, 2304, [2303]),          # the last position of the cache
    (3, 32, 8, 1024, [31, 32, 700]),   # unit boundaries
    (16, 32, 8, 8320, [4096, 8191, 5000, 6001, 4097, 7777, 8000, 4500, 6500, 7000, 5555, 4444, 8190, 6666, 5432, 7890]),
    (8, 32, 32, 1152, [1024 + i for i in range(8)]),   # multi-head attention: one query head per KV head
    (2, 16, 2, 512, [100, 3]),         # 8 query heads per KV head
    (2, 12, 4, 300, [299, 150]),       # 3 query heads per KV head, a cache of 300 positions
    (1, 32, 1, 1024, [700]),           # multi-query: 4 groups of 8 query heads read the one KV head
    (2, 24, 1, 512, [100, 3]),         # 24 query heads per KV head: 3 groups of 8
    (1, 20, 2, 256, [255]),            # 10 per KV head: groups of 8 and 2
])
def test_cluster_decode_attention_matches_oracle(lib, B, H, Hk, S, pos0):
    """The tensor-core decode attention (one cluster per KV-head group, pieces merged
    in distributed shared memory) against the oracle: the probabilities enter P V in
    bf16 and the output is rounded to bf16, as in the flash kernel."""
    import llama_decoder_forward_fwd_b200 as L
    d = 128
    q, kc, vc, ref = _attn_case(B, 1, H, Hk, d, S, pos0, torch.bfloat16, 31)
    out = torch.full((B, 1, H * d), float("nan"), dtype=torch.bfloat16, device=DEV)
    p = torch.tensor(pos0, dtype=torch.int32, device=DEV)
    for _ in range(2):
        L.llm_op_attention_decode_cluster(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out)
    torch.cuda.synchronize()
    err = np.abs(O.f64(out.cpu()) - ref)
    assert err.max() <= 8e-3 * float(vc.abs().max()), err.max()


def test_split_kv_attention_batch_16_long_caches_matches_oracle(lib):
    """The split-KV kernel at the batched-decode workload's shape (16 sequences,
    caches of 4096-8192 positions): the plan splits by length (12 splits of more
    than 704 keys per CTA) rather than to fill the GPU."""
    import llama_decoder_forward_fwd_b200 as L
    import seeded_inputs as S
    w = S.WORKLOADS["llama3-8b-bf16-b16-kv4k8k-g128"]
    B, H, Hk, d, S_max = w.batch, 32, 8, 128, 8192
    lens = S.make_kv_prefill(w.shape, w.seed, B, *w.kv_len_range, layers=[])[0]
    pos0 = [min(int(x), S_max - 1) for x in lens]
    q, kc, vc, ref = _attn_case(B, 1, H, Hk, d, S_max, pos0, torch.bfloat16, 41)
    out = torch.full((B, 1, H * d), float("nan"), dtype=torch.bfloat16, device=DEV)
    p = torch.tensor(pos0, dtype=torch.int32, device=DEV)
    ws = torch.empty(L.llm_op_attention_decode_workspace(B, 1, H, Hk, d), dtype=torch.uint8, device=DEV)
    L.llm_op_attention_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out, ws)
    torch.cuda.synchronize()
    err = np.abs(O.f64(out.cpu()) - ref)
    assert err.max() <= 6e-3 * float(vc.abs().max()), err.max()
