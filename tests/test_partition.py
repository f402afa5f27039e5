"""Host-side decode work partition (kvq_decode_partition), no GPU: the CTA
ranges cover every (row, item) once, in order, start quantized ranges on a
stage boundary, and balance the stage weights to within one chunk."""
import pytest

from quantized_kv_cache_18_b200 import workloads as W
from quantized_kv_cache_18_b200.cache import config_from_workload, decode_partition, make_config

WS, WW = 2, 3   # weights of a stage of quantized items and of a window chunk


def stage_items(cfg):
    """Quantized items per stage: the decode kernels' consumer warps take one
    32-token block each (12 KIVI warps in either formulation, 11 TURBO)."""
    if cfg.scheme != 0:
        return 11
    return 12 // (cfg.group // 32)


def check(cfg, n_groups, r, sms):
    item0, n_items = decode_partition(cfg, n_groups, r, sms)
    rows = cfg.batch * cfg.num_kv_heads
    A = cfg.anchor_tokens if cfg.scheme != 0 else 0
    n_w = -(-r // 32) + A // 32
    assert n_items == n_groups + n_w
    n = len(item0) - 1
    assert 1 <= n <= min(sms, 160)
    assert item0[0] == 0 and item0[-1] == rows * n_items
    assert all(b > a for a, b in zip(item0, item0[1:])), "a CTA owns no item"
    sg = stage_items(cfg)
    S = -(-n_groups // sg)
    # each CTA's range starts at a chunk start: a stage boundary of a row's
    # quantized items, or a window chunk
    for it in item0[:-1]:
        k = it % n_items
        assert k >= n_groups or k % sg == 0, (it, k)
    # chunk weights per CTA
    def weight(lo, hi):
        w = 0
        for it in range(lo, hi):
            k = it % n_items
            if k < n_groups:
                w += WS if k % sg == 0 else 0
            else:
                w += WW
        return w
    U = rows * (S * WS + n_w * WW)
    ws = [weight(a, b) for a, b in zip(item0, item0[1:])]
    assert sum(ws) == U
    assert max(abs(w - U / n) for w in ws) <= WW, (ws, U / n)
    return n


@pytest.mark.parametrize("name", ["tiny", "8b2", "8b4", "70b", "tq", "tqm"])
@pytest.mark.parametrize("sms", [148, 132, 7, 1])
def test_workload_partitions(name, sms):
    w = W.WORKLOADS[name]
    cfg = config_from_workload(w)
    tq = w.seq_len - w.residual - (w.anchor_tokens if w.scheme == "turbo" else 0)
    n_groups = max(0, tq) // w.group
    for r in (w.residual, w.residual + 1, w.residual + w.group - 1):
        check(cfg, n_groups, r, sms)


@pytest.mark.parametrize("g,G,bits", [(1, 32, 2), (2, 32, 2), (4, 64, 4), (8, 32, 2), (8, 64, 4)])
@pytest.mark.parametrize("n_groups,r", [(0, 0), (0, 1), (0, 160), (1, 0), (3, 31), (257, 32), (4096, 128), (13, 1)])
def test_edge_partitions(g, G, bits, n_groups, r):
    cfg = make_config("kivi", bits, G, 128, 128, 2, 2 * g, 3, max(4096 * G + 512, 1 << 20), "bf16")
    if n_groups == 0 and r == 0:
        # nothing to attend: the host partition refuses it instead of dividing by zero
        with pytest.raises(ValueError):
            decode_partition(cfg, n_groups, r, 148)
        return
    check(cfg, n_groups, r, 148)


def test_one_cta_per_chunk_at_most():
    # tiny work: never more CTAs than chunks
    cfg = make_config("kivi", 2, 32, 32, 64, 1, 2, 1, 4096, "fp16")
    item0, _ = decode_partition(cfg, 1, 1, 148)
    assert len(item0) - 1 <= 2


def test_rejects_bad_arguments():
    cfg = make_config("kivi", 2, 32, 128, 128, 8, 32, 1, 8192, "bf16")
    with pytest.raises(ValueError):
        decode_partition(cfg, -1, 0, 148)
    with pytest.raises(ValueError):
        decode_partition(cfg, 4, 0, 0)


def test_unsupported_group_is_rejected():
    cfg = make_config("kivi", 2, 32, 128, 128, 2, 12, 1, 8192, "bf16")   # GQA group of 6
    with pytest.raises(ValueError):
        decode_partition(cfg, 4, 0, 148)
