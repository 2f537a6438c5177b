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
    """Per step: FP8 key cache + scales, query-side indexer inputs, the score
    row written and read, the indices written and read, the gathered latent
    rows, bf16 q and the fp32 output with its LSE."""
    for name, S, want_mb in [("decode_32k", 32768, 472.4), ("decode_64k", 65536, 766.1)]:
        cfg = inputs.CONFIGS[name]
        B, k = 64, 2048
        total = (B * S * (128 + 4) + B * 64 * (128 + 4 + 4) + 2 * B * S * 4 + 2 * B * k * 4
                 + B * k * 576 * 2 + B * 128 * 576 * 2 + B * 128 * (512 * 4 + 4))
        got = bench.decode_bytes(cfg)["total"]
        assert got == total
        assert abs(got / 1e6 - want_mb) < 0.5
