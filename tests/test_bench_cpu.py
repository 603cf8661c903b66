"""bench.py's reporting arithmetic, on synthetic profile records (no GPU):
the dominant kernel class, achieved = algorithmic bytes (FLOPs) / time,
frac = achieved / peak, the block step against 8 TB/s, and the DRAM
traffic records of the current chain and SM-pair GEMM kernels."""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from kv_cache_decode_dualcache_b200 import synth  # noqa: E402


def _stat(name, launches, ms, gbytes=0.0, tflop=0.0):
    return {"name": name, "launches": launches, "total_ms": ms, "bytes": gbytes * 1e9,
            "flops": tflop * 1e12}


def test_hbm_bound_class_dominates():
    stats = [_stat("chain.step", 33, 100.0, gbytes=300.0),          # 3 TB/s
             _stat("gemm.qkv.full", 32, 40.0, tflop=20.0),
             _stat("attn.step", 32, 10.0, gbytes=0.5)]
    r = bench.roofline_from_profile(stats, 6000.0, 1400.0, "measured",
                                    {"step": 123.0, "full": 77.0})
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - 3000.0) < 1e-6
    assert abs(r["frac"] - 0.5) < 1e-9
    assert r["traffic"] == 123.0 and r["launches"] == 33
    assert abs(r["share_of_kernel_time"] - 100.0 / 150.0) < 1e-3
    assert r["algorithmic_bytes_per_launch"] == round(300e9 / 33)
    assert r["kernel"].startswith("chain_kernel") and r["peak_source"] == "measured"
    # per class: bytes and FLOPs over its own time
    assert r["classes"]["chain.step"] == {"launches": 33, "ms": 100.0, "GBps": 3000.0,
                                          "TFps": 0.0}
    assert r["classes"]["gemm.qkv.full"]["TFps"] == 500.0
    assert r["classes"]["attn.step"]["GBps"] == 50.0


def test_tensor_bound_class_dominates():
    stats = [_stat("chain.step", 33, 10.0, gbytes=30.0),
             _stat("gemm.qkv.full", 32, 40.0, tflop=20.0),
             _stat("gemm.ffn_up.full", 32, 60.0, tflop=40.0)]
    r = bench.roofline_from_profile(stats, 6000.0, 1400.0, "measured",
                                    {"step": 123.0, "full": None})
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["kernel"].startswith("gemm_tc2_kernel") and r["launches"] == 64
    assert abs(r["achieved"] - 60.0 / 0.1) < 1e-6       # 60 TFLOP in 100 ms
    assert abs(r["frac"] - 600.0 / 1400.0) < 1e-4
    assert r["traffic"] is None                          # no capture of this class
    r = bench.roofline_from_profile(stats, 6000.0, 1400.0, "measured",
                                    {"step": 123.0, "full": 77.0})
    assert r["traffic"] == 77.0


def test_block_step_roofline_of_the_headline_workload():
    wl = synth.WORKLOADS["llada8b-p256-g256"]
    r = bench.block_step_roofline(wl, 4.0, 6000.0)
    # weights of one block step (bf16) + K and V of all 512 positions
    want = 2 * synth.step_weight_params(wl.shape) + 32 * 512 * 32 * 128 * 2 * 2
    assert r["bytes_per_step"] == want
    assert r["ms_per_step"] == 4.0 and r["achieved_GBps"] == round(want / 4e-3 / 1e9, 1)
    assert abs(r["frac_of_8TBps"] - want / 4e-3 / 8e12) < 1e-4
    assert abs(r["frac_of_measured"] - want / 4e-3 / 6e12) < 1e-4


def test_traffic_records_follow_their_kernel_sources():
    for record, source, key in (("chain_traffic.txt", "chain.cu", "step"),
                                ("gemm_tc2_traffic.txt", "gemm_tc2.cu", "full")):
        path = os.path.join(ROOT, "profiles", record)
        rec = dict(l.split(":", 1) for l in open(path) if ":" in l and not l.startswith("#"))
        src = open(os.path.join(ROOT, "kv_cache_decode_dualcache_b200", "csrc", source),
                   "rb").read()
        got = bench.traffic_records()[key]
        if rec["source_sha256"].strip() == hashlib.sha256(src).hexdigest():
            assert got == float(rec["bytes_per_launch"])
        else:                       # kernel changed since the counters were taken
            assert got is None


def test_reference_arm_line_on_a_small_model():
    # the float64 oracle's whole generate of the tiny workload, timed on the
    # host cores: one JSON line with the contract's keys, not an estimate
    import json
    import subprocess
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["estimated"] is False
    assert line["unit"] == "tokens/s" and line["value"] > 0 and line["higher_is_better"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == "tiny"


def test_oracle_sample_clamps_its_depth_to_the_model():
    # a model with fewer layers than the 4-layer sample runs all of them,
    # unscaled
    wl = synth.WORKLOADS["tiny"]
    w = {k: v.cpu() for k, v in synth.make_weights(wl.shape, device="cpu").items()}
    r = bench.oracle_sample(wl, w, (4, 10))
    assert r["layers"] == wl.shape.n_layers == 2
    assert abs(r["t_refresh_s"] + r["t_step_s"] - r["sample_s"]) < 1e-12
    assert 0 < r["t_refresh_s"] < 60 and 0 < r["t_step_s"] < 60
    # generated tokens over the weighted, depth-scaled step times
    assert abs(r["tok_s"] - 64 / (4 * r["t_refresh_s"] + 10 * r["t_step_s"])) < 1e-9 * r["tok_s"]
    # a deeper model: the first 4 layers, scaled to its depth
    deep = synth.with_layers(synth.TINY, 6)
    wl6 = type(wl)(**{**wl.__dict__, "shape": deep})
    w6 = {k: v.cpu() for k, v in synth.make_weights(deep, device="cpu").items()}
    r6 = bench.oracle_sample(wl6, w6, (4, 10))
    assert r6["layers"] == 4
    assert abs(r6["t_refresh_s"] + r6["t_step_s"] - 1.5 * r6["sample_s"]) < 1e-12


def test_generate_roofline_of_the_headline_workload():
    wl = synth.WORKLOADS["llada8b-p256-g256"]
    spb = [1, 3, 3, 3, 4, 4, 4, 4]                      # 8 refresh + 18 block steps
    r = bench.generate_roofline(wl, spb, 1000.0, 6549.0, 1381.7)
    assert r["steps"] == {"full": 8, "cached": 18}
    # a block step is HBM-bound: the same bytes as block_step_roofline
    b = bench.block_step_roofline(wl, 1.0, 6549.0)["bytes_per_step"]
    assert abs(r["block_step_ms"]["nominal"] - 1e3 * b / 8e12) < 1e-3
    assert abs(r["block_step_ms"]["measured"] - 1e3 * b / 6549e9) < 1e-3
    # a full forward over L = 512 rows is tensor-bound: 2 x layer weights x L
    # + 2 x LM head x B + 4 L^2 H hd per layer
    sh = wl.shape
    head = sh.vocab * sh.d_model
    layers = synth.step_weight_params(sh) - head
    fl = 2 * layers * 512 + 2 * head * 32 + 4 * 512 * 512 * 32 * 128 * 32
    assert abs(r["full_step_ms"]["nominal"] - 1e3 * fl / 2.25e15) < 1e-3
    total = 8 * fl / 2.25e15 + 18 * b / 8e12
    assert abs(r["tokens_per_s"]["nominal"] - 256 / total) < 0.01
    assert abs(r["frac"]["nominal"] - 1000.0 / (256 / total)) < 1e-4


def test_generate_roofline_cache_modes():
    wl = synth.WORKLOADS["llada8b-p256-g256"]
    none = bench.generate_roofline(type(wl)(**{**wl.__dict__, "cache_mode": "none"}),
                                   [3] * 8, 100.0, 6549.0, 1381.7)
    assert none["steps"] == {"full": 24, "cached": 0}
    pre = bench.generate_roofline(type(wl)(**{**wl.__dict__, "cache_mode": "prefix"}),
                                  [3] * 8, 100.0, 6549.0, 1381.7)
    dual = bench.generate_roofline(wl, [3] * 8, 100.0, 6549.0, 1381.7)
    # the same step counts cost most without a cache, least with DualCache;
    # a prefix step over at most 256 rows costs a DualCache step's bytes, and
    # is HBM-bound at the nominal peaks (ridge 281 FLOP/B) but tensor-bound at
    # the measured ones (ridge 211 FLOP/B)
    assert none["tokens_per_s"]["nominal"] < pre["tokens_per_s"]["nominal"]
    assert pre["tokens_per_s"]["nominal"] == dual["tokens_per_s"]["nominal"]
    assert pre["tokens_per_s"]["measured"] < dual["tokens_per_s"]["measured"]
    assert bench.generate_roofline(synth.WORKLOADS["llada8b-batch16"], [3] * 8, 1.0, 1.0,
                                   1.0) is None
    # exact totals: cache off = 24 full forwards; prefix = per block one full
    # forward and two steps over rows [s, L) (tensor-bound at the measured
    # peaks once the rows pass the ridge)
    full = [none["full_step_ms"][k] for k in ("nominal", "measured")]
    assert abs(none["tokens_per_s"]["nominal"] - 256 / (24 * full[0] * 1e-3)) < 1.0
    sh = wl.shape
    head = sh.vocab * sh.d_model
    layers = synth.step_weight_params(sh) - head
    step_bytes = 2 * (layers + head) + 2 * 2 * sh.n_layers * 512 * sh.n_kv_heads * sh.head_dim

    def t(rows):
        fl = 2.0 * layers * rows + 2.0 * head * 32 + 4.0 * rows * 512 * 32 * 128 * 32
        return max(step_bytes / 6549e9, fl / 1381.7e12)
    want = sum(t(512) + 2 * t(512 - (256 + 32 * b)) for b in range(8))
    assert abs(pre["tokens_per_s"]["measured"] - 256 / want) < 0.01
