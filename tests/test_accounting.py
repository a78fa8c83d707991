"""Byte accounting of the benchmark (host logic, no GPU)."""

from mixed_precision_kv_loopkv_b200.accounting import decode_bytes, step_bytes


def test_per_token_head_bytes():
    """4-bit: 128 bytes per token-head plus 32 per selected token (D = 128);
    2-bit: 96; bf16: 512; plus query, output and block-table entries."""
    fixed = 2 * 128 * 2 + 4 * (4096 // 16)
    assert decode_bytes("q4", 128, 4096, 0) - fixed == 128 * 4096
    assert decode_bytes("q4", 128, 4096, 100) - fixed == 128 * 4096 + 32 * 100
    assert decode_bytes("q2", 128, 4096, 0) - fixed == 96 * 4096
    assert decode_bytes("bf16", 128, 4096, 0) - fixed == 512 * 4096
    assert decode_bytes("q4", 64, 0, 0) == 256


def test_unfinished_key_group_reads_exact_tail():
    # 40 tokens: one quantised key group (32) + 8 exact bf16 keys
    got = decode_bytes("q2", 128, 40)
    want = 512 + 4 * 3 + 32 * 32 + 32 * 128 * 4 // 32 + 8 * 256 + 40 * 32 + 40 * 16
    assert got == want


def test_step_bytes_resolves_reuse():
    plan = ["reuse", "q2", "q4", "q4"]          # 2 loops x 2 layers
    b1 = step_bytes(plan, 2, 2, 128, 1, [64], [64])
    want = 2 * decode_bytes("q4", 128, 64) + decode_bytes("q2", 128, 64) + decode_bytes("q4", 128, 64)
    assert b1 == want


def test_grouped_queries_count_the_cache_once_per_group():
    """G query heads on one KV head: the cache and the union's low-plane rows
    once per KV head, queries and outputs once per query head."""
    from mixed_precision_kv_loopkv_b200.accounting import decode_bytes, step_bytes
    plan, lens = ["q4", "q2"], [100, 33]
    sel = [[[5, 5, 5, 5, 7, 7, 7, 7]] * 2, [[0] * 8] * 2]
    got = step_bytes(plan, 2, 1, 128, 8, lens, lens, sel, group=4)
    want = 0
    for b, n in enumerate(lens):
        for s4 in (5, 7):
            want += decode_bytes("q4", 128, n, s4) + 3 * 2 * 128 * 2
        want += 2 * (decode_bytes("q2", 128, n) + 3 * 2 * 128 * 2)
    assert got == want
    # one query per KV head: the per-head sum
    assert step_bytes(plan, 2, 1, 128, 2, lens, lens, [[[5, 7]] * 2, [[0, 0]] * 2]) == sum(
        decode_bytes(k, 128, n, s) for k, ss in (("q4", (5, 7)), ("q2", (0, 0))) for n in lens for s in ss)


def test_reuse_current_token_adds_its_exact_row():
    from mixed_precision_kv_loopkv_b200.accounting import step_bytes
    plan = ["reuse", "q2", "q4", "q4"]
    base = step_bytes(plan, 2, 2, 128, 2, [64], [64])
    cur = step_bytes(plan, 2, 2, 128, 2, [64], [64], reuse_current=True)
    assert cur - base == 2 * 4 * 128          # one reuse cell, two heads, K + V bf16 rows
