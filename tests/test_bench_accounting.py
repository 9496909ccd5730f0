"""The bench's accounting (host logic, no GPU): algorithmic bytes and flops
counted from first principles, the reference arm's JSON line, and the
warm-up rule."""
import importlib.util
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_work_from_first_principles():
    """B=128 rows, k=2048 keys: each selected 576-value bf16 row once, the
    queries (128 heads x (128 + 64) bf16), the int32 indices, the output
    (128 x 128 bf16) and wkv_b (128 x 256 x 512 bf16) once; flops of the fold
    and W_UV (2 x 128 x 128 x 512 each per row) and of the scores and mix
    (2 x 128 x (576 + 512) per key)."""
    b = _bench()
    B, k = 128, 2048
    rows = B * k * 576 * 2
    queries = B * 128 * (128 + 64) * 2
    idx = B * k * 4
    out = B * 128 * 128 * 2
    wkv_b = 128 * 256 * 512 * 2
    flops = B * (2 * (2 * 128 * 128 * 512) + k * 2 * 128 * (576 + 512))
    assert b.algorithmic_work(B, k) == (rows + queries + idx + out + wkv_b, flops)
    assert b.algorithmic_work(B, k) == (347_078_656, 77_309_411_328)
    assert b.core_kernel_work(B, k) == (B * k * (1152 + 4), B * k * 278_528)


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "1",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0 and line["n_gpus"] == 1
    assert line["unit"] == "head*keys/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["top_k"] == 2048 and line["config"]["batch_per_gpu"] == 8


def test_fewer_than_three_warmup_steps_are_rejected():
    r = subprocess.run([sys.executable, "bench.py", "--warmup", "2"], cwd=ROOT,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 2 and "warmup" in r.stderr


def test_kernel_hash_ignores_comments_only():
    """The profiled-traffic key changes with the attend kernel's code, not
    with its comments."""
    import bench
    rels = ("sparse_head_latent_absorbed_b200/csrc/decode.cu",
            "sparse_head_latent_absorbed_b200/csrc/common.cuh")
    texts = [open(os.path.join(bench.ROOT, r), encoding="utf-8").read() for r in rels]
    base = bench.kernel_source_sha(texts)
    assert base == bench.kernel_source_sha()
    commented = [texts[0] + "\n// a note\n\n", texts[1].replace("\n", "  // x\n", 1)]
    assert bench.kernel_source_sha(commented) == base
    changed = [texts[0].replace("kRescaleThreshold = 8.0f", "kRescaleThreshold = 7.0f"), texts[1]]
    assert changed[0] != texts[0]
    assert bench.kernel_source_sha(changed) != base
