"""Host-side pieces of bench.py: the algorithmic FLOP and byte counts against the figures worked
out by hand for the named workloads, the packed workload's sequence table, and the source hash
that keeps a DRAM traffic record valid only for unchanged kernel code."""
import os

import pytest

import bench
from gated_deltanet_chunked_prefill_b200.workloads import CONFIGS

# (workload, forward GFLOP, forward MB, backward GFLOP, backward MB), from the chunked-algorithm
# convention (dense GEMMs at 2 flop/MAC, the inverse at C^3/3 MAC per chunk, every input read once
# and every output written once), computed by hand per configuration.
TABLE = [
    ("dense_bf16", 47.96, 278.4, None, None),
    ("long_gqa_bf16", 174.66, 813.7, None, None),
    ("varlen_bf16", 191.84, 1130.4, None, None),
    ("bwd_bf16", None, None, 98.78, 479.2),
]


@pytest.mark.parametrize("name,fg,fmb,bg,bmb", TABLE)
def test_algorithmic_counts(name, fg, fmb, bg, bmb):
    w = CONFIGS[name]
    if fg is not None:
        assert bench.flops(w, True, False) / 1e9 == pytest.approx(fg, abs=0.01)
        assert bench.alg_bytes(w, True, False) / 1e6 == pytest.approx(fmb, abs=0.1)
    if bg is not None:
        assert bench.flops(w, False, True) / 1e9 == pytest.approx(bg, abs=0.01)
        assert bench.alg_bytes(w, False, True) / 1e6 == pytest.approx(bmb, abs=0.1)


def test_per_token_flops():
    """182,955 flop per token and v-head forward, 376,832 backward (d = 128, MHA)."""
    w = CONFIGS["dense_bf16"]
    units = w.B * w.T * w.Hv
    assert bench.flops(w, True, False) / units == pytest.approx(182955, abs=1)
    assert bench.flops(w, False, True) / units == pytest.approx(376832, abs=1)


def test_packed_workload_is_packed():
    """The packed workload carries its 24 sequence lengths, so the bench passes cu_seqlens."""
    w = CONFIGS["varlen_bf16"]
    assert w.num_seqs == 24 and sum(w.lengths) == w.T == 65536 and w.B == 1
    assert any(n % 64 for n in w.lengths)           # at least one ragged last chunk


def test_decode_bytes():
    """State in and out (fp32), v, o, g, beta per v-head, q, k per q/k head."""
    assert bench.decode_bytes(1, 1, 1, 128, 128) == 2 * 128 * 128 * 4 + 2 * 128 * 2 + 6 + 2 * 128 * 2
    assert bench.decode_bytes(256, 16, 16, 128, 128) == 541089792


def test_source_hash_ignores_comments(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src = tmp_path / "k.cu"
    src.write_text("int f() { return 1; }  // one\n/* block\n comment */\n")
    h1 = bench.sources_sha(["k.cu"])
    src.write_text("// a new note\nint f() { return 1; }  // changed comment\n\n")
    assert bench.sources_sha(["k.cu"]) == h1
    src.write_text("int f() { return 2; }\n")
    assert bench.sources_sha(["k.cu"]) != h1
    assert bench.sources_sha(["missing.cu"]) is None
    assert os.path.exists(src)


def test_cuda_core_kernel_bytes():
    """The tiny fp32 workload (B1 H2 T256, dk = dv = 64, fp32, h0 = 0), by hand. Forward: q, k, v
    and o at 256 x 2 x 64 x 4 = 131,072 B each, g and beta 256 x 2 x 8 = 4,096 B, hT 2 x 64 x 64 x 4
    = 32,768 B: 561,152 B. Backward: q k v dO in, dq dk dv out (7 x 131,072), g beta in and dg dbeta
    out (2 x 4,096), dhT in and dh0 out (2 x 32,768): 991,232 B."""
    kb = bench.kernel_alg_bytes(CONFIGS["tiny_fp32"])
    assert CONFIGS["tiny_fp32"].h0_std is None
    assert kb["gdn_fwd_simt_kernel"] == [561152]
    assert kb["gdn_bwd_simt_kernel"] == [991232]


def _bench(args, **env):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py")] + args, cwd=root, capture_output=True,
                       text=True, timeout=600, env={**os.environ, **env})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_line():
    """`--impl reference` (the oracle on the host cores; no GPU needed) prints one line with the
    GPU arm's metric, unit and direction, its own cpu_baseline and an e2e with no copies."""
    (d,) = _bench(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["higher_is_better"] is True and d["value"] > 0 and d["steps"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    """Under a multi-rank launch only rank 0 runs and prints the reference line."""
    assert _bench(["--impl", "reference", "--steps", "1", "--warmup", "0"], RANK="1", WORLD_SIZE="2") == []
