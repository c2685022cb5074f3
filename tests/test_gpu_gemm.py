"""Zero-copy GEMM study (C = A . B, A in HBM, B in mapped host memory) against the fp64
oracle on sampled entries. Bound per entry: |C - ref| <= 2e-4 * sum_k |a b| + 1e-6
(fp32 accumulation of bf16 products; the recursive-summation bound K * 2^-24 is far larger
than the blocked tensor-core accumulation error at these K)."""
import numpy as np
import pytest
import torch

import workloads as WL

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import kv_cache_offload_b200 as dkv
    from oracle import dkv_oracle as O
else:
    dkv = O = None

VARIANTS = ["CPU_AWARE", "NAIVE_ZERO_COPY", "STAGED_SWAP", "DEVICE"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_offload_b200.build import build
    build()


def _run(variant, A, Bt, M, N, K):
    v = getattr(dkv, "DKV_GEMM_" + variant)
    Ad = A.cuda()
    C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(dkv.dkv_gemm_workspace_bytes(v, M, N, K), dtype=torch.uint8, device="cuda")
    if variant == "DEVICE":
        dkv.dkv_gemm(v, Ad, Bt.cuda(), C, ws, M, N, K)
        torch.cuda.synchronize()
        return C
    hb = dkv.dkv_host_alloc_mapped(N * K, torch.bfloat16)
    try:
        hb.tensor.copy_(Bt.reshape(-1))
        dkv.dkv_gemm(v, Ad, hb.dev_ptr, C, ws, M, N, K)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == 0
        return C
    finally:
        hb.close()


def _check(C, A, Bt, M, N, seed=0, count=2048):
    i, j = WL.gemm_sample_pairs(M, N, count, seed)
    ab, bb = WL.bf16_bits(A), WL.bf16_bits(Bt)
    ref = O.gemm_entries(ab, bb, i.numpy(), j.numpy())
    bound = O.gemm_abs_bound(ab, bb, i.numpy(), j.numpy())
    got = C[i.cuda(), j.cuda()].double().cpu().numpy()
    err = np.abs(got - ref)
    assert np.all(err <= 2e-4 * bound + 1e-6), float((err / (bound + 1e-30)).max())


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (384, 512, 640), (1024, 768, 1152)])
def test_gemm_variants_match_oracle_and_each_other(M, N, K):
    A = WL.uniform_bf16((M, K), 100 + M)
    Bt = WL.uniform_bf16((N, K), 200 + N)
    outs = {v: _run(v, A, Bt, M, N, K) for v in VARIANTS}
    _check(outs["CPU_AWARE"], A, Bt, M, N)
    for v in VARIANTS[1:]:
        # the per-tile arithmetic is identical; only the tile order and B's location differ
        assert torch.equal(outs[v], outs["CPU_AWARE"]), v


def test_gemm_rejects_unsupported_shapes():
    A = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    Bt = torch.zeros((200, 64), dtype=torch.bfloat16, device="cuda")
    C = torch.zeros((128, 200), dtype=torch.float32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_gemm(dkv.DKV_GEMM_DEVICE, A, Bt, C, ws, 128, 200, 64)
    assert e.value.code == dkv.DKV_ERR_UNSUPPORTED


def test_gemm_full_size_cpu_aware_sampled():
    cfg = WL.GEMM_CONFIGS["gemm"]
    A, Bt = WL.make_gemm_inputs(cfg, seed=0)
    C = _run("CPU_AWARE", A, Bt, cfg.M, cfg.N, cfg.K)
    _check(C, A, Bt, cfg.M, cfg.N, seed=0, count=4096)
