"""Host-side pieces of bench.py (CPU only): the paged-cache setup of ``--paged``.

``to_pages`` moves a contiguous latent cache into a page pool at shuffled positions; the
oracle's ``gather_pages`` (pinned by its own scatter/gather check) must give the contiguous
cache back, so the paged bench times the same attention as the contiguous one.
"""
import numpy as np
import torch

import bench
import oracle


def test_to_pages_round_trip_through_the_oracle_gather():
    B, Hkv, L, r, ps = 3, 2, 300, 16, 128          # 300 tokens: 3 pages, the last one partial
    g = torch.Generator().manual_seed(5)
    cache = torch.randn((B, Hkv, L, r), generator=g).to(torch.bfloat16)
    mp = -(-L // ps)
    perm = torch.randperm(B * mp, generator=g)
    pool, bt = bench.to_pages(cache, ps, perm)
    assert pool.shape == (B * mp, Hkv, ps, r) and pool.dtype == torch.bfloat16
    assert bt.shape == (B, mp) and bt.dtype == torch.int32
    assert sorted(bt.flatten().tolist()) == list(range(B * mp))   # every pool page used once
    lens = np.array([L, 129, 0], np.int32)
    back = oracle.gather_pages(pool.to(torch.float64).numpy(), bt.numpy(), lens, L)
    want = cache.to(torch.float64).numpy()
    for b in range(B):
        assert np.array_equal(back[b, :, :lens[b]], want[b, :, :lens[b]])
    # the padding past L in the last page is zero
    last = pool[int(bt[0, mp - 1])]
    assert torch.all(last[:, L - (mp - 1) * ps:] == 0)


def test_to_pages_exact_pages_need_no_padding():
    cache = torch.arange(2 * 1 * 256 * 8, dtype=torch.float32).reshape(2, 1, 256, 8)
    perm = torch.tensor([3, 0, 2, 1])
    pool, bt = bench.to_pages(cache, 128, perm)
    assert bt.tolist() == [[3, 0], [2, 1]]
    assert torch.equal(pool[3, 0], cache[0, 0, :128]) and torch.equal(pool[1, 0], cache[1, 0, 128:])


def test_row_bytes_of_each_cache_form():
    """Bytes per (token, sequence, KV head): bf16 rows, int8 rows with two fp32 scales, and
    per-head keys plus one joint value row shared by the Hkv heads."""
    import stief_inputs as si
    w = si.WORKLOADS["llama3_8b_32k"]
    assert bench.row_bytes_fn(w)(64, 64) == 256
    assert bench.row_bytes_fn(w, int8=True)(64, 64) == 64 + 64 + 8
    assert bench.row_bytes_fn(w, joint=True)(64, 64) == 2 * 64 + 2 * 64 / w.Hkv
    # fewer bytes per step: at least as many replicas to keep the rotation above 3x L2
    assert bench.replica_count(w, joint=True) >= bench.replica_count(w)
    total = bench.replica_count(w, joint=True) * sum(
        bench.row_bytes_fn(w, joint=True)(rK, rV) * w.B * w.Hkv * w.L for rK, rV in w.layer_ranks())
    assert total >= bench.ROTATE_BYTES or bench.replica_count(w, joint=True) == bench.MAX_REPLICAS


def test_cpu_baseline_reports_cores_and_cpu_model():
    """The oracle's timed baseline names what it ran on (a short budget keeps this quick)."""
    import stief_inputs as si
    res = bench.cpu_baseline(si.WORKLOADS["tiny"], budget_s=0.5)
    assert res["kind"] == "oracle" and res["cores"] >= 1 and res["value"] > 0
    assert isinstance(res["cpu_model"], str) and res["cpu_model"]


def test_algorithmic_bytes_follow_the_footprint_formula():
    """The bench's algorithmic bytes per decode are the latent footprint 2 (r_K + r_V) bytes per
    (token, KV head, sequence): 64 MiB at batch 1, 8 KV heads, 32768 tokens, ranks 64/64;
    160 MiB at 131072 tokens, ranks 32/48; 512 MiB at batch 64, 4096 tokens, ranks 64/64;
    256 KiB for one KV head at 1024 tokens.  Against the full bf16 cache (2 * d * 2 bytes per
    token and KV head) the ranks 64/64 keep half the bytes."""
    import stief_inputs as si
    W = si.WORKLOADS
    per_launch = lambda w: bench.row_bytes_fn(w)(*w.layer_ranks()[0]) * w.B * w.Hkv * w.L
    assert per_launch(W["llama3_8b_32k"]) == 64 * 2**20
    assert per_launch(W["llama31_8b_128k"]) == 160 * 2**20
    assert per_launch(W["prefill_b64"]) == 512 * 2**20
    assert per_launch(W["tiny"]) == 256 * 2**10
    w = W["llama3_8b_32k"]
    assert bench.row_bytes_fn(w)(64, 64) * 2 == 2 * w.d * 2


def test_step_call_names_the_api_call_of_each_mode():
    class A:
        int8 = int4 = latent = paged = joint = unfused = False
    cases = [({}, "stief_append_decode"), ({"unfused": True}, "stief_decode_attention"),
             ({"latent": True}, "stief_decode_latent"), ({"int8": True}, "stief_decode_attention_q8"),
             ({"int8": True, "int4": True}, "stief_decode_attention_q4"),
             ({"paged": True}, "stief_append_decode_paged"),
             ({"joint": True}, "stief_decode_attention_joint_v"),
             ({"joint": True, "latent": True}, "stief_decode_latent_joint_v")]
    for flags, want in cases:
        a = A()
        for k, v in flags.items():
            setattr(a, k, v)
        assert bench.step_call(a) == want
