"""GPU parity: sqa_attn_fwd_rows (a block of query rows at a global offset against all keys).

Against the float64 oracle's row mode on the same seeded inputs (the forward's
bar), and, at offsets that are multiples of the 128-row tile, against rows of
the whole-sequence sqa_attn_fwd: the shards of a sequence (the per-rank step of
sequence sharding) reassemble the full output within the same bar. Not bit for
bit: a launch whose last wave is partial splits the keys of those tiles over
two CTAs, each rounding P to bf16 against its own half's running maximum, and
which tiles land in that wave depends on the launch's size, so a shard and the
whole sequence can differ by P's rounding.
"""
import numpy as np
import pytest

import oracle
from helpers import assert_close, attn_inputs, bf16_tensor_to_f64, default_scale, run_attn, to_device_bf16

pytestmark = pytest.mark.gpu


def run_rows(qb_block, kb, vb, q_offset, causal, scale):
    import torch
    import reduced_query_head_b200 as sqa
    B, n, H_q, d = qb_block.shape
    N, H_kv = kb.shape[1], kb.shape[2]
    out = torch.full((B, n, H_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sqa.sqa_attn_fwd_rows(to_device_bf16(qb_block), to_device_bf16(kb), to_device_bf16(vb), out, B, n, N, q_offset,
                          H_q, H_kv, d, int(causal), scale)
    st = sqa.sqa_device_status()
    assert st == sqa.SQA_OK, sqa.sqa_status_string(st)
    return out


CASES = [
    # B, N_k, q_offset, N_q, H_q, H_kv, d
    (1, 1000, 0, 1000, 8, 4, 64),     # the whole sequence
    (1, 1000, 333, 200, 8, 4, 64),    # an interior block off the tile grid
    (2, 777, 700, 77, 16, 1, 64),     # the last rows, MQA with 16 heads stacked
    (1, 513, 1, 511, 12, 3, 128),     # all but the first row, d = 128
    (1, 1000, 123, 300, 8, 2, 128),   # d = 128 block whose rows start off the 80-key step grid
    (3, 300, 150, 1, 6, 4, 64),       # one row, uneven groups
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dNk%doff%dNq%dHq%dHkv%dd%d" % c)
def test_rows_against_oracle(case, causal):
    B, N, off, n, H_q, H_kv, d = case
    scale = default_scale(d)
    qb, kb, vb = attn_inputs(B, N, H_q, H_kv, d, seed=70)
    got = bf16_tensor_to_f64(run_rows(np.ascontiguousarray(qb[:, off:off + n]), kb, vb, off, causal, scale))
    rows = np.array([b * N + off + t for b in range(B) for t in range(n)])
    want = oracle.attention_rows(oracle.widen_bf16(qb.reshape(B * N, H_q, d)[rows]), oracle.widen_bf16(kb),
                                 oracle.widen_bf16(vb), rows, N, causal, scale)
    assert_close(got.reshape(B * n, H_q, d), want, str(case), out_rounding=True)


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_shards_reassemble_the_whole_sequence(world, causal):
    import torch
    from reduced_query_head_b200.dist import sequence_blocks
    B, N, H_q, H_kv, d = 1, 2048, 16, 4, 64
    qb, kb, vb = attn_inputs(B, N, H_q, H_kv, d, seed=71)
    full = run_attn(qb, kb, vb, causal, 0.125)
    assembled = torch.full_like(full, float("nan"))
    for r in range(world):
        for a, b in sequence_blocks(N, r, world, causal):
            assert a % 128 == 0 and b % 128 == 0
            assembled[:, a:b] = run_rows(np.ascontiguousarray(qb[:, a:b]), kb, vb, a, causal, 0.125)
    want = oracle.attention(oracle.widen_bf16(qb), oracle.widen_bf16(kb), oracle.widen_bf16(vb), causal, 0.125)
    assert_close(bf16_tensor_to_f64(assembled), want, "sharded over %d" % world, out_rounding=True)
    assert_close(bf16_tensor_to_f64(full), want, "whole sequence", out_rounding=True)
