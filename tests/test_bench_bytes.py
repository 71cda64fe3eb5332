"""The algorithmic byte counts behind bench.py's roofline figures, against
their closed forms (no GPU needed)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    argv, sys.argv = sys.argv, ["bench.py"]
    try:
        import bench
    finally:
        sys.argv = argv
    return bench


def test_forward_bytes_per_token_head():
    b = _bench()
    th = 4 * 4096 * 16                                  # token-heads of the B4 T4096 H16 workload
    state = 2 * 4 * 16 * 128 * 128 * 4 + 16 * 128 * 4    # S read and written, gamma_stat read
    # q k z b (d_k) and v w g (d_v) in bf16, fp32 log-decay, bf16 y: 2560 B
    assert b.fwd_bytes(4, 4096, 16, 128, 128, 2) == th * 2560 + state == 679485440
    # no z: 2304 B; beta for b and w: 2050 B; plus one fp32 decay and no z: 1286 B
    assert b.fwd_bytes(4, 4096, 16, 128, 128, 2, z=False) == th * 2304 + state
    assert b.fwd_bytes(4, 4096, 16, 128, 128, 2, beta=True) == th * 2050 + state
    assert b.fwd_bytes(4, 4096, 16, 128, 128, 2, z=False, beta=True, decay_tok=True) == th * 1286 + state


def test_decode_and_backward_bytes():
    b = _bench()
    # decode: state read + written per head, tokens (4 d_k + 3 d_v bf16), fp32 log-decay, bf16 y
    per_head = 2 * 128 * 128 * 4 + 7 * 128 * 2 + 128 * 4 + 128 * 2
    assert b.decode_bytes(64, 16, 128, 128, 2) == 64 * 16 * per_head + 16 * 128 * 4 == 136847360
    # backward per token-head: the forward inputs without y (2304 B), fp32 dL/dy (512 B) and
    # eight fp32 gradients (4096 B); per head S_in, dL/dS_out read and dL/dS_in written
    th = 4 * 4096 * 16
    assert b.bwd_bytes(4, 4096, 16, 128, 128, 2) == th * (2304 + 512 + 4096) + 3 * 64 * 65536 + 2 * 16 * 512
