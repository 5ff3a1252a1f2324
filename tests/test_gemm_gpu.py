"""GPU tests of the block's projection GEMM (ssm_proj_gemm: C = A . W^T on
tcgen05, bf16 operands, fp32 accumulation, bf16 output), the in_proj and
out_proj of "Axon-SSM: selective state space model", "Algorithm" diagram.

Reference: the products of the stored bf16 values summed in float64 on the
CPU, rounded once to bf16. The kernel accumulates the same products in fp32
(K <= 7680 terms: relative error ~1e-6, far below a bf16 step), so the two
roundings agree except for rare one-step flips: relative L2 <= 1e-3 is asked.
The kernel runs on CTA pairs (256 x 256 tiles, two-SM MMAs). Shapes cover
ragged M, N and K tails (the second CTA of a pair past M), more tiles than
pairs (each persistent pair taking several whole tiles, alternating its two
accumulators, then a run of K chunks), tiles cut along K between pairs (few
tiles, long K: fp32 partials summed in pair order by the contributor that
completes the count, so the output is the same on every call) and the
block's layer shapes.
"""
import numpy as np
import pytest
import torch

from selective_state_space_depthwise_b200 import _lib, api

pytestmark = pytest.mark.gpu

TOL_GEMM = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def operands(M, N, K, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    A = torch.randn((M, K), generator=g).to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g) * K ** -0.5).to(torch.bfloat16)
    return A, W


def reference(A, W, rows=None):
    a = A.double().numpy() if rows is None else A[rows].double().numpy()
    return torch.from_numpy(a @ W.double().numpy().T).to(torch.bfloat16).double().numpy()


def rel_l2(got, want):
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


SHAPES = [(1, 8, 8), (100, 136, 72), (300, 520, 200), (129, 264, 64), (257, 1000, 1032)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in SHAPES])
def test_gemm_ragged_shapes(shape):
    M, N, K = shape
    A, W = operands(M, N, K, seed=M + N + K)
    C = api.proj_gemm(A.cuda(), W.cuda())
    torch.cuda.synchronize()
    e = rel_l2(C.double().cpu().numpy(), reference(A, W))
    print(f"gemm {M}x{N}x{K}: rel-L2 {e:.2e}")
    assert e <= TOL_GEMM


@pytest.mark.parametrize("shape", [(2000, 256 * 29 - 24, 200), (2000, 256 * 26 - 24, 200)],
                         ids=["whole_then_cut", "whole_only"])
def test_gemm_many_tiles_per_cta(shape):
    """More output tiles than CTA pairs: each persistent pair takes several
    whole tiles, so both TMEM accumulators alternate and the grouped raster
    wraps (8 row blocks x 29 or 26 column blocks). 232 tiles (3.1 a pair):
    two rounds of whole tiles, then a run of tiles cut along K; 208 tiles
    (2.8 a pair): three rounds of whole tiles, the last one partly idle."""
    M, N, K = shape
    assert (api.proj_gemm_workspace_bytes(M, N, K) > 0) == (N == 256 * 29 - 24)
    A, W = operands(M, N, K, seed=N)
    C = api.proj_gemm(A.cuda(), W.cuda())
    torch.cuda.synchronize()
    e = rel_l2(C.double().cpu().numpy(), reference(A, W))
    print(f"gemm {M}x{N}x{K}: rel-L2 {e:.2e}")
    assert e <= TOL_GEMM


@pytest.mark.parametrize("shape", [(256, 512, 4096), (200, 264, 1000)], ids=["16_way", "4_way_ragged"])
def test_gemm_tiles_cut_along_k(shape):
    """Few output tiles and a long K: every tile is cut along K between CTA
    pairs (16 and 4 contributors a tile) whose fp32 partials the last
    contributor sums. Every element against the reference, twice with the
    same workspace (its tile counters are zeroed by each call), and the two
    outputs bit-equal (the sum runs in pair order whoever finishes last)."""
    M, N, K = shape
    assert api.proj_gemm_workspace_bytes(M, N, K) > 0  # this shape cuts tiles
    A, W = operands(M, N, K, seed=K)
    ws = torch.empty(api.proj_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    want = reference(A, W)
    outs = []
    for _ in range(2):
        C = api.proj_gemm(A.cuda(), W.cuda(), workspace=ws)
        torch.cuda.synchronize()
        e = rel_l2(C.double().cpu().numpy(), want)
        print(f"gemm cut tiles {M}x{N}x{K}: rel-L2 {e:.2e}")
        assert e <= TOL_GEMM
        outs.append(C)
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("which", ["in_proj", "out_proj"])
def test_gemm_layer_shapes_sampled_rows(which):
    """The block's projections at the Axon layer shape (2048 tokens, D = 2560,
    E = 7680): every column of 96 sampled rows against the float64 reference,
    the full output finite, and two calls bit-equal (out_proj cuts its tiles
    between two CTA pairs; the one that finishes last adds the other's partial
    to its own accumulator, which gives the same sum either way)."""
    M, D, E = 2048, 2560, 7680
    N, K = (2 * E, D) if which == "in_proj" else (D, E)
    A, W = operands(M, N, K, seed=7 if which == "in_proj" else 8)
    C = api.proj_gemm(A.cuda(), W.cuda())
    C2 = api.proj_gemm(A.cuda(), W.cuda())
    torch.cuda.synchronize()
    assert torch.isfinite(C).all()
    assert torch.equal(C, C2)
    rows = np.sort(np.random.default_rng(3).choice(M, 96, replace=False))
    rows[0], rows[-1] = 0, M - 1
    e = rel_l2(C[torch.from_numpy(rows).cuda()].double().cpu().numpy(), reference(A, W, rows))
    print(f"{which} {M}x{N}x{K}: rel-L2 {e:.2e} over {len(rows)} rows")
    assert e <= TOL_GEMM


def test_gemm_rejects_bad_arguments():
    A = torch.zeros((16, 12), dtype=torch.bfloat16, device="cuda")  # K = 12 is not a multiple of 8
    W = torch.zeros((8, 12), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.SsmError) as err:
        api.proj_gemm(A, W)
    assert err.value.status == _lib.SSM_ERR_INVALID_ARG
