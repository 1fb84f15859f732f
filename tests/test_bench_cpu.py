"""The benchmark's reference arm (the CPU oracle timed on the host) prints the
one JSON line the benchmark contract asks for; runs without a GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert out.returncode == 0
    assert not [l for l in out.stdout.splitlines() if l.startswith("{")]


def test_every_layer_stage_has_a_launch_count_and_a_cost_model():
    """Each stage name a layer can produce (default, shared expert apart,
    gather, fused combine) is known to the benchmark's launch count and
    per-stage cost model, for every configuration."""
    sys.path.insert(0, ROOT)
    import torch
    import bench
    from moe_inputs import CONFIGS
    from mixture_experts_layer_limited_b200 import MoELayer, LayerSpec
    for name, cfg in CONFIGS.items():
        if cfg.dtype != "bf16":
            continue
        spec = LayerSpec.from_config(cfg)
        H, E, I, Is, T = cfg.H, cfg.E, cfg.I, cfg.I_s, 4
        z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
        model = bench.stage_model(cfg)
        for kw in ({}, {"fuse_shared": False}, {"gather": True}, {"fuse_combine": True}, {"fuse_ffn": True},
                   {"fuse_ffn": False}):
            # shapes only: stages() builds the launch closures without running them
            lay = MoELayer(spec, z(E, 8), z(1, 1), z(1, 1), z(1, 1) if Is else None,
                           z(1, 1) if Is else None, None, T, tiled_weights=False, **kw)
            names = [n for n, _ in lay.stages(z(T, H))] + ["bias_update"]
            for n in names:
                assert n in bench.LAUNCHES and n in model, (name, kw, n)
                assert bench.launches_of(n, cfg) >= 1


def test_one_launch_ffn_is_chosen_from_512_routed_rows_per_expert():
    """bf16 layers with a shared expert run both GEMMs in one launch when the
    routed rows average at least two full token blocks per expert (T*k >=
    512*E), as two launches below; fuse_ffn True / False force either."""
    sys.path.insert(0, ROOT)
    import torch
    from moe_inputs import get_config
    from mixture_experts_layer_limited_b200 import MoELayer, LayerSpec
    cfg = get_config("v3")
    spec = LayerSpec.from_config(cfg)
    z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    E, k, H = cfg.E, cfg.k, cfg.H
    T_max = 512 * E // k                                  # exactly two token blocks per expert
    for fuse, T, want in ((None, T_max, "ffn"), (None, T_max - 1, "gate_up"), (True, 8, "ffn"),
                          (False, T_max, "gate_up")):
        lay = MoELayer(spec, z(E, 8), z(1, 1), z(1, 1), z(1, 1), z(1, 1), None, T_max, fuse_ffn=fuse,
                       tiled_weights=False)
        names = [n for n, _ in lay.stages(z(T, H))]
        assert want in names, (fuse, T, names)


def test_cpu_sample_holds_every_token_of_the_hottest_and_coldest_expert():
    """The CPU baseline's sample: at least n_min tokens, every token of the
    expert with the most rows and of the one with the fewest (non-empty)
    rows, no token twice."""
    sys.path.insert(0, ROOT)
    import types
    import numpy as np
    import torch
    import bench
    import oracle
    from moe_inputs import get_config
    rng = np.random.default_rng(5)
    T, k, E = 4096, 8, 64
    L = rng.standard_normal((T, E)).astype(np.float32)
    L[:, 3] += 2.0                                   # a hot expert
    L[:, 17] -= 3.0                                  # a cold one
    ids = oracle.route_from_logits(L, k, 1, 1, "softmax", False, 1.0).ids
    off, src, _ = oracle.permute(ids, E)
    layer = types.SimpleNamespace(offsets=torch.from_numpy(off.astype(np.int32)),
                                  src_token=torch.from_numpy(src.astype(np.int32)))
    cfg = types.SimpleNamespace(T=T, k=k)
    toks, hot, n_hot, cold, n_cold = bench.cpu_sample_tokens(layer, cfg, 1024)
    counts = np.diff(off)
    assert hot == int(np.argmax(counts)) and n_hot == counts.max()
    assert cold == int(np.argmin(np.where(counts > 0, counts, 10 ** 9))) and n_cold > 0
    assert len(toks) >= 1024 and len(set(toks.tolist())) == len(toks)
    for e in (hot, cold):
        assert set(src[off[e]:off[e + 1]].tolist()) <= set(toks.tolist())


def test_profiled_traffic_matches_workload_stage_and_source(monkeypatch):
    """roofline.traffic comes from the committed one-launch DRAM summaries
    (profiles/*_traffic.txt): the V3 gate/up launch, the E4M3 decode layer's
    gate/up stage and the skewed layer's one-launch FFN, each only for its
    own workload and stage, near
    the algorithmic bytes, and none once the GEMM source differs from the one
    captured."""
    sys.path.insert(0, ROOT)
    import bench
    v3 = bench.profiled_traffic("gate_up", "v3")
    f8 = bench.profiled_traffic("gate_up", "v3_fp8_decode")
    assert v3 is not None and f8 is not None
    assert 1.0 <= v3 / 16450060288 < 1.2          # the split experts re-read part of their weights
    assert 0.85 < f8 / 7566786560 <= 1.0          # experts without tokens are never read
    sk = bench.profiled_traffic("ffn", "v3_skewed")
    assert sk is not None and 1.0 <= sk / 33508294656 < 1.2
    assert bench.profiled_traffic("down", "v3") is None
    v2 = bench.profiled_traffic("gate_up", "v2lite")
    assert v2 is not None and 0.9 < v2 / 970981376 < 1.1
    assert bench.profiled_traffic("gate_up", "tiny") is None
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic("gate_up", "v3") is None
