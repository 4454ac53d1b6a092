"""Host-side accounting of bench.py (no GPU): the algorithmic bytes that the
roofline fraction divides by, and the rule that reports ncu traffic only for
the workload and kernel sources it was captured on."""
import bench
import workloads


def test_step_bytes_hand_count():
    # L 1, H 2 (C = 2 heads), G 2, D 64, bf16; 100 entries before eviction on
    # 8 pages, 60 kept, 5 rows moved by compaction
    cfg = workloads.small_config(L=1, H=2, G=2, D=64, B=1, kv_dtype="bf16")
    k_all = 2 * 64 * 100          # K of every entry (dense logits for the dropped mass)
    v_kept = 2 * 64 * 60          # V of the kept entries
    q_out = 2 * 4 * 2 * 2 * 64    # fp32 queries in, outputs out: C * G rows of D
    lse_dm = 2 * 4 * 2 * 2        # fp32 lse and dropped mass per query row
    tables = (4 + 2) * 8          # block-table entry + keep word per page
    attn = k_all + v_kept + q_out + lse_dm + tables
    assert bench.attn_bytes(cfg, 100, 60, 8) == attn == 22_608
    row = 2 * 2 * 64 + 8          # K + V + position + log-retention
    select = 8 * 100              # position + log-retention of every entry
    moves = 2 * row * 5           # each moved row read and written
    append = 2 * row              # one appended row per head
    assert bench.step_bytes(cfg, 100, 60, 8, evict=True, moves=5) == attn + select + moves + append == 26_576
    # a non-evicting step reads no selection metadata and moves nothing
    assert bench.step_bytes(cfg, 100, 100, 8, evict=False) == bench.attn_bytes(cfg, 100, 100, 8) + append


def test_step_bytes_fp32_rows():
    cfg = workloads.small_config(L=1, H=1, G=1, D=128, B=1, kv_dtype="f32")
    row = 2 * 4 * 128 + 8
    assert bench.step_bytes(cfg, 10, 4, 1, moves=3) - bench.attn_bytes(cfg, 10, 4, 1) == 8 * 10 + 2 * row * 3 + row


def test_traffic_only_for_the_captured_workload_and_sources():
    files = bench.TRAFFIC_SOURCES
    cur = bench.sources_sha(files)
    llama, qwen = workloads.CONFIGS["llama32k"], workloads.CONFIGS["qwen8k"]
    rec = {"sources_sha256": cur, "workload": "llama32k", "bytes_per_launch": 123.0}
    assert bench.kernel_traffic(llama, None, rec, files) == 123.0
    assert bench.kernel_traffic(qwen, None, rec, files) is None
    stale = dict(rec, sources_sha256="0" * 16)
    assert bench.kernel_traffic(llama, None, stale, files) is None
    assert bench.kernel_traffic(llama, 7.0, stale, files) == 7.0    # --traffic overrides
    # the two kernels' records hash different source sets
    assert bench.sources_sha(bench.ATTN_TRAFFIC_SOURCES) != cur
