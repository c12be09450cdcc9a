"""The analytic bytes behind the bench's roofline numbers, against the
per-request figures worked out by hand for the small layer (batch 256, 64
heads, head_dim 64, d_state 128, 8 groups, bf16 inputs, fp32 state):
state 4 H P N = 2,097,152 B; one buffered entry (x row, B row, dt) =
H P 2 + G N 2 + 4 H = 10,496 B; one token's inputs (x, B, C, dt) =
H P 2 + 2 G N 2 + 4 H = 12,544 B; y = 4 H P = 16,384 B."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from hybrid_model_ssm_replay_b200.inputs import WORKLOADS  # noqa: E402


def test_small_layer_bytes():
    sh = WORKLOADS["small_b256"]["shape"]
    b = bench.shape_bytes(sh)
    assert (b["state"], b["entry"], b["inputs"], b["y"]) == (2_097_152, 10_496, 12_544, 16_384)
    # decode at buffer position t: state + t entries read + the new entry + inputs + y
    assert bench.decode_bytes_per_request(sh, 0) == 2_097_152 + 10_496 + 12_544 + 16_384
    assert bench.decode_bytes_per_request(sh, 15) - bench.decode_bytes_per_request(sh, 0) == 15 * 10_496
    # flush of 16 entries: read + write the state, read the entries
    assert bench.flush_bytes_per_request(sh, 16) == 2 * 2_097_152 + 16 * 10_496
    # conventional: read + write the state every token
    assert bench.conv_bytes_per_request(sh) == 4_223_232
    # one interval of replay (16 decodes + flush) per token, and its ratio to the conventional step
    per_tok = (sum(bench.decode_bytes_per_request(sh, t) for t in range(16)) +
               bench.flush_bytes_per_request(sh, 16)) / 16
    assert per_tok == 2_487_936
    assert abs(4_223_232 / per_tok - 1.697) < 1e-3


def test_bytes_saved_ratio():
    """Conventional bytes per token over replay bytes per token: 1.697 with
    the separate flush; with the fused fold the filling token writes the
    folded state (2,097,152 B) instead of its buffer entry (10,496 B) and no
    flush runs: (35,444,736 + 2,097,152 - 10,496) / 16 = 2,345,712 B per
    token, ratio 1.800."""
    sh = WORKLOADS["small_b256"]["shape"]
    assert abs(bench.bytes_saved_ratio(sh) - 4_223_232 / 2_487_936) < 1e-12
    assert sum(bench.decode_bytes_per_request(sh, t) for t in range(16)) == 35_444_736
    assert abs(bench.bytes_saved_ratio(sh, fused=True) - 4_223_232 * 16 / (35_444_736 + 2_097_152 - 10_496)) < 1e-12
    assert abs(bench.bytes_saved_ratio(sh, fused=True) - 1.800) < 1e-3
