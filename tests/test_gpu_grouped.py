"""GPU grouped (MoE) decode GEMV against the oracle: stacked experts
[E, N, K/2] as in imp docs/quantization.md (MoE layers), synthetic routing."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import assert_within_tolerance, guarded_empty

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import gemm_decode_nvfp4_b200 as m
    assert torch.cuda.is_available()
    return m


def _experts(E, N, K, seed):
    qs, ss = zip(*[workloads.random_codes(N, K, seed + e) for e in range(E)])
    q = np.stack([a.numpy() for a in qs])
    s = np.stack([b.numpy() for b in ss])
    g = (np.arange(1, E + 1, dtype=np.float32) * np.float32(0.003))
    return q, s, g


def _run(nv, X, q, s, g, experts, tokens):
    P, N = len(experts), q.shape[1]
    Y, check = guarded_empty((P, N), torch.bfloat16)
    nv.gemv_grouped(X.cuda(), torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(g).cuda(),
                    torch.tensor(experts, dtype=torch.int32, device="cuda"),
                    torch.tensor(tokens, dtype=torch.int32, device="cuda"), Y)
    check()
    return Y


@pytest.mark.parametrize("E,N,K,T", [(16, 1536, 2048, 1),   # ring kernel, top-8 of 16 for one token
                                     (8, 700, 1024, 4),     # ring, four tokens
                                     (6, 300, 1040, 3)])    # K % 256 != 0: register kernel
def test_grouped_matches_oracle(nv, E, N, K, T):
    q, s, g = _experts(E, N, K, 5 * E + N)
    X = workloads.random_bf16((T, K), 9)
    rng = np.random.default_rng(N)
    experts = [int(e) for e in rng.integers(0, E, 8)]   # repeats allowed
    tokens = [int(t) for t in rng.integers(0, T, 8)]
    y_ref, bound = oracle.linear_grouped(X, q, s, g, experts, tokens)
    Y = _run(nv, X, q, s, g, experts, tokens)
    for p in range(len(experts)):
        assert_within_tolerance(Y[p], y_ref[p], bound[p], f"problem {p} (expert {experts[p]}, token {tokens[p]})")
    nv.check_device_errors()


def test_grouped_bad_ids_zero_rows_and_report(nv):
    E, N, K = 4, 256, 1024
    q, s, g = _experts(E, N, K, 31)
    X = workloads.random_bf16((2, K), 32)
    experts, tokens = [1, E, 2, 0], [0, 1, 5, 1]        # problem 1: expert out of range; problem 2: token
    Y = _run(nv, X, q, s, g, experts, tokens)
    assert not Y[1].float().abs().sum().item() and not Y[2].float().abs().sum().item()
    y_ref, bound = oracle.linear_grouped(X, q, s, g, [1, 0], [0, 1])
    assert_within_tolerance(Y[0], y_ref[0], bound[0], "valid problem 0")
    assert_within_tolerance(Y[3], y_ref[1], bound[1], "valid problem 3")
    with pytest.raises(nv.Nvfp4Error) as err:
        nv.check_device_errors()
    assert err.value.status == 1 and "out-of-range" in str(err.value)
    nv.check_device_errors()  # the counter was cleared


def test_grouped_ids_written_by_previous_kernel(nv):
    """A kernel earlier on the stream writes the routing: the GEMV must see it."""
    E, N, K = 8, 512, 2048
    q, s, g = _experts(E, N, K, 41)
    X = workloads.random_bf16((1, K), 42)
    qd, sd, gd = torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(g).cuda()
    ids = torch.zeros(6, dtype=torch.int32, device="cuda")
    toks = torch.zeros(6, dtype=torch.int32, device="cuda")
    Y = torch.empty((6, N), dtype=torch.bfloat16, device="cuda")
    Xd = X.cuda()
    for rep in range(3):
        ids.copy_(torch.tensor([(rep + 3 * i) % E for i in range(6)], dtype=torch.int32), non_blocking=True)
        ids.add_(0)  # a device kernel writes the ids right before the GEMV
        nv.gemv_grouped(Xd, qd, sd, gd, ids, toks, Y)
        torch.cuda.synchronize()
        experts = [(rep + 3 * i) % E for i in range(6)]
        y_ref, bound = oracle.linear_grouped(X, q, s, g, experts, [0] * 6)
        for p in range(6):
            assert_within_tolerance(Y[p], y_ref[p], bound[p], f"rep {rep} problem {p}")
