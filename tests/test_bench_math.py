"""The benchmark's roofline arithmetic, against hand counts (no GPU)."""
import types

import torch

import bench
from long_context_decode_full_b200 import synth


def _workload(name, lens):
    return types.SimpleNamespace(spec=synth.WORKLOADS[name], seq_lens=torch.tensor(lens, dtype=torch.int32))


def test_step_bytes_at_256k_context():
    ab = bench.algorithmic_bytes(_workload("ctx256k_b4_bf16_paged", [262144] * 4))
    kv = 4 * 262144 * 4 * (2 * 128 * 2)          # every K and V row, bf16, 4 KV heads
    scores = 4 * (262144 - 128) * 4 * 8          # one fp32 score written and read per selectable position
    qo = 4 * 32 * 128 * 2 * 2                    # the query in, the output out
    rows = 4 * 4 * 1152 * (2 * 128 * 2)          # a sparse layer's listed rows
    assert ab["full_attention"] == kv == 2147483648
    assert ab["step"] == kv + scores + qo + 3 * (rows + qo) == 2209595392


def test_e4m3_rows_carry_their_scales_and_short_sequences_skip_scores():
    ab = bench.algorithmic_bytes(_workload("ctx1m_b1_fp8_paged", [1048576]))
    assert ab["full_attention"] == 1048576 * 4 * (2 * 128 + 8)
    # a sequence that fits window + k_global selects everything: no score traffic
    short = bench.algorithmic_bytes(_workload("decode_b8_32k_bf16", [1000] * 8))
    assert short["full_layer"] - short["full_attention"] == 8 * 32 * 128 * 2 * 2


def test_bridge_bytes():
    # hidden 4096, 4 KV heads x 128: two 4096 x 512 bf16 matrices, 4 hidden rows, 8 stored rows
    assert bench.bridge_bytes(4, 4096, 4, 128, 2, False) == 2 * 4096 * 512 * 2 + 4 * 4096 * 2 + 2 * 4 * 512 * 2
    assert bench.bridge_bytes(1, 4096, 4, 128, 1, True) == 2 * 4096 * 512 * 2 + 4096 * 2 + 2 * 512 + 2 * 4 * 4
