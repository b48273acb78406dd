"""bench.py on the host, no GPU needed: the reference arm (the oracle timed
on this host's cores) on the tiny configuration prints one JSON line with
the contract's keys; option checks; the quantised inputs' recipe."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "0", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    d = json.loads(lines[-1])
    assert d["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["value"] > 0 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_batch_override_is_refused_outside_its_modes():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--batch", "2"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 2
    assert "--batch applies to --prefill-attn and --per-head-rank only" in r.stderr


def test_quantised_bench_inputs_are_what_the_quantiser_stores(monkeypatch):
    """The benchmark's int8 / int4 caches are quantised from profile-shaped
    rows by the latent quantiser's rule, so they are a fixed point of the
    oracle's quantiser: re-quantising the dequantised rows gives the same
    codes and the same fp16 scales, bit for bit, and every group reaches
    +-qmax (its amax element).  A shrunk workload keeps it fast on CPU."""
    import numpy as np

    import bench
    import synthetic
    from oracle import quant_ref as qr
    small = synthetic.replace(synthetic.CONFIGS[3], E=512, H=4, r=256, B=2, L=300)
    monkeypatch.setitem(synthetic.CONFIGS, 3, small)
    for cache, bits in (("i8", 8), ("i4", 4)):
        inp = bench.bench_inputs(3, "cpu", cache=cache)
        w = inp["w"]
        raw = inp["cache"].numpy()
        codes = qr.unpack_int4(raw) if cache == "i4" else raw.view(np.int8)
        sc = inp["scales"].numpy()
        deq = qr.dequantize(codes, sc, w.group)
        c2, s2, over = qr.quantize(deq, bits, w.group)
        assert not over.any()
        assert np.array_equal(c2, codes)
        assert np.array_equal(s2.view(np.uint16), sc.view(np.uint16))
        qmax = 7 if bits == 4 else 127
        gmax = np.abs(codes.astype(np.int32)).reshape(codes.shape[:-1] + (-1, w.group)).max(-1)
        assert (gmax == qmax).all()
