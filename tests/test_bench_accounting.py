"""The bench's algorithmic work per step (the roofline numerators), against sums
written out by hand for three workloads (no GPU needed)."""
import bench
from long_context_token_b200 import workloads


def test_bytes_of_the_8x131072_bf16_step():
    w = workloads.WORKLOADS[2]
    ab = bench.alg_bytes(w, [131072] * 8)
    kv = 2 * 8 * 131072 * 256                 # K and V rows, 256 B each
    q, out = 8 * 16 * 128 * 2, 8 * 16 * 128 * 4
    assert ab["full"] == kv + q + out == 536_969_216
    idx = 8 * 1152 * 4
    sparse = 2 * 8 * 1152 * 256 + idx + q + out  # gathered rows, indices, queries, outputs
    assert ab["sparse"] == sparse
    assert ab["step"] == ab["full"] + idx + 3 * sparse == 551_567_360


def test_bytes_of_the_1m_fp8_h64_step():
    w = workloads.WORKLOADS[4]
    ab = bench.alg_bytes(w, [1048576])
    row = 128 + 4                              # E4M3 row plus its float32 scale
    q, out = 64 * 128 * 2, 64 * 128 * 4
    assert ab["full"] == 2 * 1048576 * row + q + out
    assert ab["step"] == ab["full"] + 1152 * 4 + 3 * (2 * 1152 * row + 1152 * 4 + q + out)


def test_flops_of_the_64_token_append_step():
    w = workloads.WORKLOADS[5]
    ab = bench.alg_bytes(w, [131072])
    # token i of 64 sees 131072 - 64 + i + 1 keys; Q.K^T and P.V: 2 * 2 * 128 flops per
    # (head, key) pair
    visible = sum(131072 - 64 + i + 1 for i in range(64))
    assert ab["full_flops"] == 4 * 128 * 16 * visible == 68_702_961_664
