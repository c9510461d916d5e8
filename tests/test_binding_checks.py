"""The Python binding hands raw pointers to the library, so every tensor must hold exactly the
elements its layout implies.  These CPU tests pass one short tensor at a time to each entry
point and expect a ValueError naming it, raised before any device work; with every size right
the first complaint is the device placement (still before any launch)."""
import pytest
import torch

import sparse_attention_backward_sfa_b200 as S

BF = torch.bfloat16


def sfa_inputs(T1=6, T2=20, N1=4, topk=5):
    q = torch.zeros(T1, N1, 512, dtype=BF)
    k = torch.zeros(T2, 1, 512, dtype=BF)
    return dict(query=q, key=k, value=k, sparse_indices=torch.zeros(T1, 1, topk, dtype=torch.int32),
                d_out=torch.zeros_like(q), out=torch.zeros_like(q),
                softmax_max=torch.zeros(T1, N1), softmax_sum=torch.ones(T1, N1),
                query_rope=torch.zeros(T1, N1, 64, dtype=BF), key_rope=torch.zeros(T2, 1, 64, dtype=BF))


KW = dict(scale=0.04, sparse_block_size=1, layout="TND", sparse_mode=0,
          actual_seq_lengths_q=torch.tensor([6], dtype=torch.int32),
          actual_seq_lengths_kv=torch.tensor([20], dtype=torch.int32))


def call_grad(a):
    return S.sfa_grad(a["query"], a["key"], a["value"], a["sparse_indices"], a["d_out"], a["out"], a["softmax_max"],
                      a["softmax_sum"], a["query_rope"], a["key_rope"], **KW)


def call_rows(a):
    acc = torch.zeros(20, 1088)
    return S.sfa_grad_rows(a["query"], a["key"], a["value"], a["sparse_indices"], a["d_out"], a["out"],
                           a["softmax_max"], a["softmax_sum"], a["query_rope"], a["key_rope"], row_begin=0, row_end=6,
                           dkv_accum=acc, **KW)


def call_fwd(a):
    return S.sfa_fwd(a["query"], a["key"], a["value"], a["sparse_indices"], a["query_rope"], a["key_rope"], **KW)


SHORT = ["key", "value", "sparse_indices", "d_out", "out", "softmax_max", "softmax_sum", "query_rope", "key_rope"]


@pytest.mark.parametrize("call,names", [(call_grad, SHORT), (call_rows, SHORT),
                                        (call_fwd, ["key", "value", "sparse_indices", "query_rope", "key_rope"])])
def test_sfa_calls_reject_short_tensors(call, names):
    for name in names:
        a = sfa_inputs()
        t = a[name]
        a[name] = t[:-1].clone()  # one leading row short: trailing dims (read by the shape inference) intact
        # a short key sets T2 itself, so the tensors sized by T2 are the ones reported
        with pytest.raises(ValueError, match=("" if name == "key" else name) + ".*elements"):
            call(a)
    with pytest.raises(ValueError, match="CUDA"):  # every size right: placement is checked last
        call(sfa_inputs())


def test_rows_rejects_a_short_accumulator():
    a = sfa_inputs()
    with pytest.raises(ValueError, match="dkv_accum.*elements"):
        S.sfa_grad_rows(a["query"], a["key"], a["value"], a["sparse_indices"], a["d_out"], a["out"], a["softmax_max"],
                        a["softmax_sum"], a["query_rope"], a["key_rope"], row_begin=0, row_end=6,
                        dkv_accum=torch.zeros(19, 1088), **KW)


def fa_inputs(T=10, N=4, Nkv=2, D=64):
    q = torch.zeros(T, N, D, dtype=BF)
    kv = torch.zeros(T, Nkv, D, dtype=BF)
    return dict(q=q, k=kv, v=kv.clone(), dy=torch.zeros_like(q), attention_in=torch.zeros_like(q),
                softmax_max=torch.zeros(T, N, 8), softmax_sum=torch.ones(T, N, 8))


def call_fa_grad(a):
    return S.fa_grad(a["q"], a["k"], a["v"], a["dy"], a["softmax_max"], a["softmax_sum"], a["attention_in"], [10],
                     [10], scale=0.125, sparse_mode=3)


def test_fa_grad_rejects_short_tensors():
    for name in ("v", "dy", "attention_in", "softmax_max", "softmax_sum"):
        a = fa_inputs()
        a[name] = a[name][:-1].clone()
        with pytest.raises(ValueError, match=f"{name}.*elements"):
            call_fa_grad(a)
    with pytest.raises(ValueError, match="CUDA"):
        call_fa_grad(fa_inputs())


def test_fa_fwd_rejects_a_short_value():
    a = fa_inputs()
    with pytest.raises(ValueError, match="v.*elements"):
        S.fa_fwd(a["q"], a["k"], a["v"][:-1].clone(), [10], [10], scale=0.125, sparse_mode=3)


def lig_inputs(T=6, N1=64, G=64, Di=128):
    q = torch.zeros(T, N1, 512, dtype=BF)
    k = torch.zeros(T, 1, 512, dtype=BF)
    return dict(query=q, key=k, query_index=torch.zeros(T, G, Di, dtype=BF), key_index=torch.zeros(T, 1, Di, dtype=BF),
                weights=torch.zeros(T, G, dtype=BF), softmax_max=torch.zeros(T, N1), softmax_sum=torch.ones(T, N1),
                softmax_max_index=torch.zeros(T), softmax_sum_index=torch.ones(T),
                query_rope=torch.zeros(T, N1, 64, dtype=BF), key_rope=torch.zeros(T, 1, 64, dtype=BF))


def call_lig(a, seq_key=True):
    cu = torch.tensor([6], dtype=torch.int64)
    return S.lig_kl_grad(a["query"], a["key"], a["query_index"], a["key_index"], a["weights"], a["softmax_max"],
                         a["softmax_sum"], a["softmax_max_index"], a["softmax_sum_index"], a["query_rope"],
                         a["key_rope"], scale=0.04, layout="TND", sparse_mode=3, actual_seq_lengths_query=cu,
                         actual_seq_lengths_key=cu if seq_key else None)


def test_lig_rejects_short_tensors_and_a_missing_key_length():
    for name in ("query_index", "key", "key_index", "weights", "query_rope", "key_rope", "softmax_max",
                 "softmax_sum", "softmax_max_index", "softmax_sum_index"):
        a = lig_inputs()
        a[name] = a[name][:-1].clone()
        with pytest.raises(ValueError, match=("" if name == "key" else name) + ".*elements"):
            call_lig(a)
    with pytest.raises(ValueError, match="actual_seq_lengths_key"):
        call_lig(lig_inputs(), seq_key=False)
    with pytest.raises(ValueError, match="CUDA"):
        call_lig(lig_inputs())
