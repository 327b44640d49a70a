"""The Python binding rejects tensors that do not match the call before anything is
launched: the kernels take raw pointers and read every tensor densely at the shape the call
implies, so a shorter, strided or differently typed tensor would otherwise be read out of
bounds or misread."""
import pytest
import torch

from gated_delta_rule_160_b200 import workloads as W

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "b", "w")


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    return g


def _args(T=130, h_qk=1, h_v=2, d=128, dtype=torch.bfloat16):
    return W.token_inputs(T, h_qk, h_v, d, d, dtype, "cuda", seed=91)


def test_prefill_arguments_are_checked(g):
    d = _args()
    fwd = lambda **kw: g.gdn2_chunk_fwd(*(kw.get(k_, d[k_]) for k_ in NAMES),
                                        **{k_: v_ for k_, v_ in kw.items() if k_ not in NAMES})
    with pytest.raises(ValueError, match="k has shape"):
        fwd(k=d["k"][:100].contiguous())
    with pytest.raises(ValueError, match="contiguous"):
        fwd(v=d["v"].transpose(0, 1).contiguous().transpose(0, 1))
    with pytest.raises(TypeError, match="log_alpha"):
        fwd(log_alpha=d["log_alpha"].to(torch.bfloat16))
    with pytest.raises(TypeError, match="b is"):
        fwd(b=d["b"].float())
    with pytest.raises(ValueError, match="S0 has shape"):
        fwd(S0=torch.zeros(1, 2, 128, 64, device="cuda"))
    with pytest.raises(TypeError, match="cu_seqlens"):
        fwd(cu_seqlens=torch.tensor([0, 130], device="cuda"))
    with pytest.raises(ValueError, match="o has shape"):
        fwd(o=torch.empty(130, 2, 64, device="cuda"))
    o, st = fwd()  # the same call with matching tensors runs
    torch.cuda.synchronize()
    assert o.shape == (130, 2, 128) and st.shape == (1, 2, 128, 128)


def test_decode_arguments_are_checked(g):
    N, n_tok = 3, 2
    d = {k_: t.view(N, n_tok, *t.shape[1:]) for k_, t in _args(T=N * n_tok).items()}
    pool = torch.zeros(5, 2, 128, 128, device="cuda")
    run = lambda **kw: g.gdn2_decode_multi(*(d[k_] for k_ in NAMES), kw.pop("pool", pool), **kw)
    with pytest.raises(TypeError, match="slots"):
        run(slots=torch.tensor([0, 1, 2], device="cuda"))
    with pytest.raises(ValueError, match="slots has shape"):
        run(slots=torch.tensor([0, 1], dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError, match="S_pool has shape"):
        run(pool=torch.zeros(5, 2, 128, 64, device="cuda"))
    with pytest.raises(TypeError, match="S_pool"):
        run(pool=pool.to(torch.bfloat16))
    o, _ = run(slots=torch.tensor([4, -1, 0], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert o.shape == (N, n_tok, 2, 128)
    S = torch.zeros(N, 2, 128, 128, device="cuda")
    x = _args(T=N)
    with pytest.raises(ValueError, match="S has shape"):
        g.gdn2_decode_step(*(x[k_] for k_ in NAMES), S[:2].contiguous())
