"""The Python binding checks every tensor argument on the host before it calls the library: a
host tensor, a wrong dtype or a tensor smaller than the call reads is rejected with no launch
(these run without a GPU: the checks come before any CUDA call)."""
import pytest
import torch

import gated_deltanet_03_b200 as g

bf, f32 = torch.bfloat16, torch.float32


def _prefill_args(T=64, Hk=1, Hv=2, D=128):
    return dict(q=torch.zeros(T, Hk, D, dtype=bf), k=torch.zeros(T, Hk, D, dtype=bf),
                v=torch.zeros(T, Hv, D, dtype=bf), a=torch.zeros(T, Hv), b=torch.zeros(T, Hv),
                A_log=torch.zeros(Hv), dt_bias=torch.zeros(Hv))


def test_host_tensors_are_rejected():
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        g.gdn_prefill_chunked(**_prefill_args())


@pytest.mark.parametrize("name,bad,err,msg", [
    ("a", torch.zeros(64, 2, dtype=torch.float64), TypeError, "a must be torch.float32"),
    ("A_log", torch.zeros(2, dtype=bf), TypeError, "A_log must be torch.float32"),
    ("k", torch.zeros(64, 1, 128, dtype=f32), TypeError, "k must be torch.bfloat16"),
    ("v", torch.zeros(64, 2, 100, dtype=bf), None, None),
    ("k", torch.zeros(63, 1, 128, dtype=bf), ValueError, "k holds 8064 elements, the call needs 8192"),
    ("b", torch.zeros(64, 1), ValueError, "b holds 64 elements, the call needs 128"),
    ("dt_bias", torch.zeros(1), ValueError, "dt_bias holds 1 elements, the call needs 2"),
])
def test_prefill_argument_checks(name, bad, err, msg):
    args = _prefill_args()
    args[name] = bad
    if err is None:       # v sets Hv and Dv: a consistent smaller v is not an error here
        with pytest.raises(ValueError, match="must be a CUDA tensor"):
            g.gdn_prefill_chunked(**args)
        return
    with pytest.raises(err, match=msg):
        g.gdn_prefill_chunked(**args)


def test_optional_tensors_are_checked():
    args = _prefill_args()
    with pytest.raises(TypeError, match="cu_seqlens must be torch.int32"):
        g.gdn_prefill_chunked(**args, cu_seqlens=torch.tensor([0, 64], dtype=torch.int64))
    with pytest.raises(ValueError, match="initial_state holds"):
        g.gdn_prefill_chunked(**args, initial_state=torch.zeros(1, 2, 128, 127))
    with pytest.raises(TypeError, match="workspace must be torch.uint8"):
        g.gdn_prefill_chunked(**args, workspace=torch.zeros(16, dtype=f32))


def test_decode_verify_commit_checks():
    B, T, Hk, Hv, D = 2, 3, 1, 2, 128
    q, k = torch.zeros(B, T, Hk, D, dtype=bf), torch.zeros(B, T, Hk, D, dtype=bf)
    v = torch.zeros(B, T, Hv, D, dtype=bf)
    a, b = torch.zeros(B, T, Hv), torch.zeros(B, T, Hv)
    A_log, dt_bias = torch.zeros(Hv), torch.zeros(Hv)
    S = torch.zeros(B, Hv, D, D)
    with pytest.raises(TypeError, match="accepted must be torch.int32"):
        g.gdn_decode_commit(q, k, v, a, b, A_log, dt_bias, S, torch.zeros(B, dtype=torch.int64))
    with pytest.raises(ValueError, match="state holds"):
        g.gdn_decode_verify(q, k, v, a, b, A_log, dt_bias, S[:1])
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        g.gdn_decode_step(q[:, 0], k[:, 0], v[:, 0], a[:, 0].contiguous(), b[:, 0].contiguous(), A_log, dt_bias, S)


def test_tail_and_gemm_checks():
    M, Hv, D = 4, 2, 128
    o, z = torch.zeros(M, Hv, D, dtype=bf), torch.zeros(M, Hv, D, dtype=f32)
    with pytest.raises(TypeError, match="z must be torch.bfloat16"):
        g.gdn_gated_rmsnorm_silu(o, z, torch.ones(D))
    with pytest.raises(ValueError, match="weight holds 64 elements, the call needs 128"):
        g.gdn_gated_rmsnorm_silu_nvfp4(o, z.to(bf), torch.ones(64), 1.0)
    Mg, N, K = 128, 64, 256
    aq, as_ = torch.zeros(Mg, K // 2, dtype=torch.uint8), torch.zeros(Mg, K // 16, dtype=torch.uint8)
    bq, bs = torch.zeros(N, K // 2, dtype=torch.uint8), torch.zeros(N, K // 16, dtype=torch.uint8)
    with pytest.raises(TypeError, match="bq must be torch.uint8"):
        g.nvfp4_gemm(aq, as_, bq.to(torch.int8), bs, 1.0)
    with pytest.raises(ValueError, match="bs holds"):
        g.nvfp4_gemm(aq, as_, bq, bs[:N // 2], 1.0)
    with pytest.raises(ValueError, match="col_alpha holds"):
        g.nvfp4_gemm_colscale(aq, as_, bq, bs, torch.ones(N - 1))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        g.nvfp4_quantize_act(torch.zeros(M, K, dtype=bf), 1.0)
