"""GPU parity of gdr2_forward_varlen (packed sequences) against the fp64 oracle.

Each packed sequence must give exactly what the oracle gives for that sequence on its
own: its own initial state, no state or product crossing from one sequence to the next.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_wy_b200 import GDR2Error, gdr2_forward, gdr2_forward_varlen, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, assert_close

pytestmark = pytest.mark.gpu


def _packed(lens, H, seed, decay_shift=2.0):
    T = int(sum(lens))
    x = I.make_forward_inputs(B=1, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=decay_shift,
                              seed=seed)
    S0 = torch.randn((len(lens), H, 128, 128), generator=torch.Generator().manual_seed(seed + 1)) * 0.1
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return x, S0, cu


def _check_against_oracle(lens, H, seed, which=None):
    x, S0, cu = _packed(lens, H, seed)
    d = x.to("cuda")
    o, S_T, _ = gdr2_forward_varlen(d.q, d.k, d.v, d.log_alpha, d.b, d.w, cu.cuda(), S0.cuda())
    gdr2_sync_status()
    n = x.as_numpy64()
    for i in (which if which is not None else range(len(lens))):
        s, e = int(cu[i]), int(cu[i + 1])
        S0_i = S0[i:i + 1].double().numpy()
        if e == s:  # an empty sequence keeps its state
            assert torch.equal(S_T[i].cpu(), S0[i]), f"empty sequence {i}: S_T != S0"
            continue
        args = [n[f][:, s:e] for f in ("q", "k", "v", "log_alpha", "b", "w")]
        o_ref, S_ref = oracle.forward(*args, S0=S0_i)
        assert_close(o[s:e][None], o_ref, TOL[torch.bfloat16], f"seq {i} (len {e - s}): o")
        assert_close(S_T[i:i + 1], S_ref, TOL[torch.bfloat16], f"seq {i} (len {e - s}): S_T")


def test_mixed_lengths_with_empty_and_ragged_sequences():
    _check_against_oracle([0, 1, 63, 64, 65, 130, 200, 17, 0, 128], H=4, seed=71)


def test_single_sequence_and_one_token_sequences():
    _check_against_oracle([300], H=2, seed=72)
    _check_against_oracle([1, 1, 1, 2, 1], H=3, seed=73)


def test_lengths_in_ascending_order():
    # the scans take the sequences longest first: here the reverse of their order in memory
    _check_against_oracle([1, 5, 63, 64, 100, 300, 700], H=3, seed=77)


def test_more_sequences_than_the_scan_order_sort_takes():
    # beyond 2048 sequences the scans take them in the given order
    rng = np.random.default_rng(78)
    lens = rng.integers(0, 24, 2100)
    lens[[5, 1000, 2099]] = [200, 130, 65]
    _check_against_oracle(lens.tolist(), H=1, seed=78, which=[0, 5, 17, 1000, 1500, 2098, 2099])


def test_equal_lengths_match_the_dense_forward_exactly():
    """B equal sequences packed, against the [B, T, H, D] forward: the same chunk and scan
    steps on the same chunks, so the same bits (including the saved chunk states)."""
    B, T, H = 3, 200, 4
    x = I.make_forward_inputs(B=B, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=74,
                              with_S0=True)
    d = x.to("cuda")
    o_d, S_d, sv_d = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, save_states=True)
    pack = lambda t: t.reshape(1, B * T, *t.shape[2:]).contiguous()  # noqa: E731
    cu = torch.arange(0, B * T + 1, T, dtype=torch.int32, device="cuda")
    o_p, S_p, sv_p = gdr2_forward_varlen(pack(d.q), pack(d.k), pack(d.v), pack(d.log_alpha), pack(d.b),
                                         pack(d.w), cu, d.S0, save_states=True)
    gdr2_sync_status()
    assert torch.equal(o_p, o_d.reshape(B * T, H, 128))
    assert torch.equal(S_p, S_d)
    nc = (T + 63) // 64
    assert torch.equal(sv_p[:B * H * nc], sv_d.reshape(B * H * nc, 128, 128))


def test_bad_cu_seqlens_is_reported_and_computes_nothing():
    x, S0, cu = _packed([64, 64], H=2, seed=75)
    d = x.to("cuda")
    bad = torch.tensor([0, 100, 64, 128], dtype=torch.int32, device="cuda")[[0, 1, 3]]  # 0, 100, 128: fine
    gdr2_forward_varlen(d.q, d.k, d.v, d.log_alpha, d.b, d.w, bad, S0[:2].cuda())
    gdr2_sync_status()  # a valid split: no error
    for bad in ([0, 100, 64], [1, 64, 128], [0, 64, 127]):  # decreasing; not from 0; not to T
        o = torch.full((128, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
        gdr2_forward_varlen(d.q, d.k, d.v, d.log_alpha, d.b, d.w,
                            torch.tensor(bad, dtype=torch.int32, device="cuda"), S0[:2].cuda(), out=o)
        with pytest.raises(GDR2Error, match="cu_seqlens"):
            gdr2_sync_status()
        assert torch.all(o == 7.0), f"{bad}: outputs were written"
    # the library is usable afterwards
    _check_against_oracle([64, 64], H=2, seed=75)


@pytest.mark.slow
def test_packed_65536_tokens_sampled_sequences():
    """65,536 tokens in 61 sequences of mixed lengths (H = 16); the oracle on six of them."""
    rng = np.random.default_rng(76)
    lens = rng.integers(1, 2048, size=60)
    lens = list(lens) + [65536 - int(lens.sum())]
    assert lens[-1] > 0
    _check_against_oracle(lens, H=16, seed=76, which=[0, 1, 17, 30, 59, 60])
