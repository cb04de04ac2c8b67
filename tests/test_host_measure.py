"""Host arithmetic of the measurement scripts (no GPU): byte counts and the
budgeted batch plan, against figures computed by hand from the workload
shapes (24 layers, 4 loops, 16 KV heads, head_dim 128, ctx 32768, group 32)."""
from kv_cache_residual_rq_b200 import capacity, synth

W = synth.ENCODE
CTX = 32768


def test_kv_bytes_per_sequence_by_hand():
    elems = 2 * 24 * 16 * CTX * 128              # K and V elements per loop
    assert synth.kv_bytes_per_sequence(W, CTX, False) == elems * 2 * 4     # 25.77 GB
    # reference bf16 + three INT2 loops (2 bits + one fp16 scale per 32)
    assert synth.kv_bytes_per_sequence(W, CTX, True) == elems * 2 + 3 * elems * (2 + 0.5) // 8


def test_compressed_reference_kv_bytes_by_hand():
    # INT8 reference (8 bits + one fp16 scale per 32) + three INT2 loops
    # (2 bits + one fp16 scale per 32 each): 16 bits per element, K and V
    elems = 2 * 24 * 16 * CTX * 128
    assert capacity.kv_bytes_per_sequence(W, CTX, "rq_cr8") == elems * 2      # 6.44 GB
    assert capacity.kv_bytes_per_sequence(W, CTX, "bf16") == elems * 2 * 4
    assert capacity.kv_bytes_per_sequence(W, CTX, "rq") == synth.kv_bytes_per_sequence(W, CTX, True)


def test_budget_plan_max_batches():
    rows, maxb = capacity.plan(W, CTX, synth.SWEEP_BATCHES, 120e9)
    assert maxb == {"bf16": 4, "rq": 12, "rq_cr8": 18}
    fits = {(s, b) for s, b, _, ok in rows if ok}
    assert fits == {("bf16", 1), ("bf16", 2), ("bf16", 4),
                    ("rq", 1), ("rq", 2), ("rq", 4), ("rq", 8), ("rq", 12),
                    ("rq_cr8", 1), ("rq_cr8", 2), ("rq_cr8", 4), ("rq_cr8", 8),
                    ("rq_cr8", 12), ("rq_cr8", 16)}


def test_step_bytes_reread_reference_each_loop():
    # one sequence: BF16 reads 4 loops of K/V; ResidualQuant reads the BF16
    # reference in each of its 4 calls plus codes and scales of 3 loops
    elems = 2 * 24 * 16 * CTX * 128
    qo = 4 * 24 * 16 * 128 * 6
    assert capacity.step_bytes(W, CTX, 1, "bf16") == elems * 2 * 4 + qo
    assert capacity.step_bytes(W, CTX, 1, "rq") == elems * 2 * 4 + 3 * elems * 5 // 16 + qo
    # compressed reference: every call reads the INT8 reference codes and
    # scales (136 bytes per token row of 128 dims), loops 1-3 add 40
    assert capacity.step_bytes(W, CTX, 1, "rq_cr8") == elems * (4 * 136 + 3 * 40) // 128 + qo


def test_call_bytes_by_hand():
    # one Ouro-shaped call: 16 x 16 heads x 4096 tokens, d 128, group 32
    from kv_cache_residual_rq_b200 import measure
    w = synth.BY_NAME["ouro1.4b_decode"]
    heads_t = 16 * 16 * 4096
    qo = 16 * 16 * 128 * 6                       # q bf16 in, out fp32
    # BF16 K/V rows, INT2 codes of K and V, one fp16 scale per 32 dims each
    assert measure.decode_bytes(w, 2) == heads_t * (2 * 256 + 2 * 32 + 2 * 8) + qo == 620953600
    assert measure.decode_bytes(w, 16) == heads_t * 2 * 256 + qo
    # compressed reference: INT8 (INT4) K/V codes and scales instead of the rows
    assert measure.cr_decode_bytes(w, 8, 2) == heads_t * (2 * 136 + 2 * 40) + qo == 369295360
    assert measure.cr_decode_bytes(w, 4, 16) == heads_t * 2 * 72 + qo
