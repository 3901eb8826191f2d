"""The Python binding rejects malformed arguments before any launch (CPU only).

The kernels trust the sizes they are given, so shapes and dtypes of every
tensor (inputs, caller-provided outputs, mask vectors) are checked first,
whatever the device; only then is each tensor required to be a contiguous
CUDA tensor on the device of q.
"""
import pytest
import torch

import column_sparse_masked_b200 as fm

B, N, HQ, HKV, D = 1, 40, 4, 2, 64


def qkv(nq=N, nk=N):
    bf = torch.bfloat16
    return (torch.zeros(B, nq, HQ, D, dtype=bf), torch.zeros(B, nk, HKV, D, dtype=bf),
            torch.zeros(B, nk, HKV, D, dtype=bf))


def masks(nk=N, hm=1):
    return [torch.zeros(B, hm, nk, dtype=torch.int32) for _ in range(4)]


@pytest.fixture(scope="module", autouse=True)
def library():
    from column_sparse_masked_b200 import build

    build.build()
    fm.load_library()


def test_well_formed_cpu_arguments_only_fail_on_the_device():
    q, k, v = qkv()
    with pytest.raises(TypeError, match="CUDA"):
        fm.fwd(q, k, v, *masks())
    o, lse = torch.zeros_like(q), torch.zeros(B, HQ, N)
    with pytest.raises(TypeError, match="CUDA"):
        fm.bwd(q, k, v, o, lse, torch.zeros_like(q), *masks())


@pytest.mark.parametrize("which", ["q3d", "k_d", "v_shape", "q_dtype"])
def test_forward_rejects_bad_qkv(which):
    q, k, v = qkv()
    if which == "q3d":
        q = q[0]
    elif which == "k_d":
        k = torch.zeros(B, N, HKV, D + 64, dtype=torch.bfloat16)
    elif which == "v_shape":
        v = torch.zeros(B, N + 1, HKV, D, dtype=torch.bfloat16)
    else:
        q = q.float()
    with pytest.raises((TypeError, ValueError)):
        fm.fwd(q, k, v, *masks())


def test_forward_rejects_mask_of_wrong_length_or_dtype():
    q, k, v = qkv()
    with pytest.raises(ValueError, match="lts"):
        fm.fwd(q, k, v, *masks(nk=N + 1))
    m = masks()
    m[2] = m[2].long()
    with pytest.raises(TypeError, match="uts"):
        fm.fwd(q, k, v, *m)


def test_forward_rejects_outputs_of_wrong_shape():
    q, k, v = qkv()
    with pytest.raises(ValueError, match="o must"):
        fm.fwd(q, k, v, *masks(), out=(torch.zeros(B, N, HQ, D - 1, dtype=torch.bfloat16), torch.zeros(B, HQ, N)))
    with pytest.raises(ValueError, match="lse"):
        fm.fwd(q, k, v, *masks(), out=(torch.zeros_like(q), torch.zeros(B, N, HQ)))


def test_backward_rejects_bad_lse_dout_and_outputs():
    q, k, v = qkv()
    o, lse, do = torch.zeros_like(q), torch.zeros(B, HQ, N), torch.zeros_like(q)
    with pytest.raises(ValueError, match="lse"):
        fm.bwd(q, k, v, o, torch.zeros(B, HQ, N + 1), do, *masks())
    with pytest.raises(ValueError, match="dout"):
        fm.bwd(q, k, v, o, lse, do[:, :-1], *masks())
    with pytest.raises(ValueError, match="dk"):
        fm.bwd(q, k, v, o, lse, do, *masks(), out=(torch.zeros_like(q), torch.zeros_like(q), torch.zeros_like(v)))
