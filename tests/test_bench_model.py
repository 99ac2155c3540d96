"""The bench's algorithmic byte model (the numerator of every roofline
fraction), checked against a separately written closed form: bytes per
(slot, head) and token averaged over one merge cycle, with d = d_k = d_v,
fp32 state and bf16 inputs (2 bytes):

  eager:    8 d^2 (state read + write) + io + gates
  deferred: 4 d^2 (state read) + 4 d^2 / M (merge write) + io + gates
            + e (M - 1) / M (entries appended) + e (M - 1) / 2 (entries replayed)

io = 3 d (q, k, v) + d (o) elements of 2 bytes; gates GDN 8, KDA 4 d + 4,
RWKV6 4 d; entry e = 2 d (a_i) + d (b_i: 4 bytes, RWKV6 2) + Lam_i (GDN 4,
else 4 d).  The RWKV6 bonus u is read once per launch (4 d H bytes)."""
import pytest

import bench


def closed_form(op, d, M):
    io = 4 * d * 2
    gates = {"gdn": 8, "kda": 4 * d + 4, "rwkv6": 4 * d}[op]
    if M == 1:
        return 8 * d * d + io + gates
    e = 2 * d + d * (2 if op == "rwkv6" else 4) + (4 if op == "gdn" else 4 * d)
    return 4 * d * d + 4 * d * d / M + io + gates + e * (M - 1) / M + e * (M - 1) / 2


@pytest.mark.parametrize("op,B,H,d", [("gdn", 256, 32, 128), ("kda", 128, 32, 128), ("rwkv6", 128, 64, 64),
                                      ("gdn", 3, 5, 64)])
@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 33])
def test_step_bytes_match_closed_form(op, B, H, d, M):
    tokens = 4 * M
    per_token = bench.step_bytes(op, B, H, d, M, tokens) / tokens
    want = closed_form(op, d, M) * B * H
    if op == "rwkv6":
        want += 4 * d * H      # the bonus, once per launch
    assert per_token == pytest.approx(want, rel=1e-12)


def test_headline_bytes():
    """GDN B=256 H=32 d=128: 1082 MB per token eager, 640 MB at M = 8."""
    assert bench.step_bytes("gdn", 256, 32, 128, 1, 1) / 1e6 == pytest.approx(1082.2, abs=0.1)
    assert bench.step_bytes("gdn", 256, 32, 128, 8, 8) / 8 / 1e6 == pytest.approx(640.1, abs=0.1)


@pytest.mark.parametrize("op,d", [("gdn", 128), ("kda", 128), ("rwkv6", 64)])
@pytest.mark.parametrize("M", [1, 4, 8, 16])
def test_write_bytes_per_token(op, d, M):
    """Writes per (slot, head) and token: eager writes the state and o every
    token; the deferred path writes o and an entry on M - 1 tokens, and o and
    the state on the merge token."""
    H = 7
    o = 2 * d
    if M == 1:
        want = 4 * d * d + o
    else:
        e = 2 * d + d * (2 if op == "rwkv6" else 4) + (4 if op == "gdn" else 4 * d)
        want = ((M - 1) * (o + e) + (o + 4 * d * d)) / M
    assert bench.write_bytes_per_token(op, 1, H, d, M) == pytest.approx(H * want, rel=1e-12)


def _count_chunk_flops(op, d, C):
    """Flops of one C-token chunk of one head, counted operation by operation
    with loops (a multiply-add counts 2), divided by C."""
    f = 0
    # dense products with the state: [C x d] times [d x d], and the update
    # [d x C] times [C x d]
    dense = 3 if op != "rwkv6" else 2
    f += dense * C * d * d * 2
    for t in range(C):
        for s in range(t + 1):
            if op == "rwkv6":
                f += 2 * d                       # P[t][s]: a dot product, or the diagonal's u (.) k . r
                f += 2 * d                       # P V: row t takes P[t][s] v_s
            else:
                if s < t:
                    f += 2 * d                   # A[t][s]
                f += 2 * d                       # P[t][s]
                f += 2 * d                       # P B
        if op != "rwkv6":
            f += 2 * t * (2 * d)                 # forward substitution, 2d right-hand-side columns
    return f / C


@pytest.mark.parametrize("op", ["gdn", "kda", "rwkv6"])
@pytest.mark.parametrize("d,C", [(64, 32), (128, 16), (128, 32), (8, 4)])
def test_chunk_prefill_flops(op, d, C):
    assert bench.chunk_prefill_flops(op, d, C) == _count_chunk_flops(op, d, C)


@pytest.mark.parametrize("op,d", [("kda", 128), ("rwkv6", 64)])
@pytest.mark.parametrize("M", [4, 8, 16])
def test_step_bytes_with_f16_log_gates(op, d, M):
    """fp16 per-key log-gates: every entry carries 2 d bytes less (the Lam_i
    term 4 d becomes 2 d), appended once and replayed (M - 1) / 2 times on
    average per token; nothing else changes.  KDA d = 128: 1280 -> 1024 bytes
    per entry; RWKV6 d = 64: 512 -> 384."""
    B, H, tokens = 3, 5, 4 * M
    full = bench.step_bytes(op, B, H, d, M, tokens) / tokens
    half = bench.step_bytes(op, B, H, d, M, tokens, lb=2) / tokens
    saved_per_entry = 2 * d
    assert full - half == pytest.approx(B * H * saved_per_entry * ((M - 1) / M + (M - 1) / 2), rel=1e-12)
    assert bench.entry_bytes(op, d, d, lb=2) == {"kda": 1024, "rwkv6": 384}[op]
