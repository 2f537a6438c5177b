"""The algorithmic work bench.py divides by: flop and byte counts checked
against brute-force enumeration on small shapes and against closed forms
written independently at the headline sizes."""
import bench
from sparse_attention_long_fp8_b200 import inputs


def _brute_pairs(L, k):
    visible = sum(t + 1 for t in range(L))
    selected = sum(min(k, t + 1) for t in range(L))
    return visible, selected


def test_visible_and_selected_pairs_match_enumeration():
    for L, k in [(1, 4), (7, 3), (100, 64), (300, 2048)]:
        cfg = inputs.custom_config("prefill_4k", n_q=L, n_kv=L, topk=k, name="acc")
        vis, sel = _brute_pairs(L, k)
        assert bench.visible_pairs(cfg) == vis
        assert bench.selected_rows(cfg) == sel


def test_headline_flop_counts():
    """Prefill at L = 65536: 2 H^I d^I per causal pair for the indexer, and
    2 H (D_qk + D_v) per selected (query, key) pair for the attention."""
    cfg = inputs.CONFIGS["prefill_64k"]
    L, k = 65536, 2048
    pairs = L * (L + 1) / 2
    sel = k * (k + 1) / 2 + (L - k) * k
    assert abs(bench.indexer_flops(cfg) - 2 * 64 * 128 * pairs) < 1
    assert abs(bench.attn_flops(cfg) - 2 * 128 * (576 + 512) * sel) < 1
    assert 35.1e12 < bench.indexer_flops(cfg) < 35.3e12
    assert 36.7e12 < bench.attn_flops(cfg) < 36.9e12


def test_decode_bytes_at_both_contexts():
    """Per step: FP8 key cache + scales, query-side indexer inputs (codes,
    scale, weight), the indices, the gathered latent rows, bf16 q and the
    fp32 output with its LSE; no score round trip (the scope table's
    ~456 MB at 32768 and ~733 MB at 65536)."""
    for name, S, want_mb in [("decode_32k", 32768, 455.1), ("decode_64k", 65536, 731.9)]:
        cfg = inputs.CONFIGS[name]
        B, k = 64, 2048
        total = (B * S * (128 + 4) + B * 64 * (128 + 4 + 4) + B * k * 4
                 + B * k * 576 * 2 + B * 128 * 576 * 2 + B * 128 * (512 * 4 + 4))
        got = bench.decode_bytes(cfg)["total"]
        assert got == total
        assert abs(got / 1e6 - want_mb) < 0.5


def test_sampled_oracle_rows_are_evenly_spaced_and_distinct():
    cfg = inputs.CONFIGS["prefill_64k"]
    for n, off in [(16, 0.5), (16, 0.01), (272, 0.99), (1, 0.5)]:
        rows = bench.oracle_sample_rows(cfg, n, off)
        assert len(rows) == n and rows.min() >= 0 and rows.max() < cfg.n_q
        assert (abs((rows[1:] - rows[:-1]) - cfg.n_q / n) <= 1).all()


def test_warmup_loss_flops():
    cfg = inputs.CONFIGS["prefill_4k"]
    pairs = 4096 * 4097 // 2
    fl = bench.warmup_loss_flops(cfg)
    assert fl["probs_bf16"] == 2.0 * 128 * 576 * pairs
    assert fl["scores_fp8"] == 2.0 * 64 * 128 * pairs
    assert fl["grads_fp32"] == 2 * fl["scores_fp8"]
