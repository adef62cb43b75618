"""Host-side logic of bench.py on CPU: algorithmic byte counts, the multi-rank
max-over-ranks reduction (gloo, world size 2), the reference arm's rank rule,
and the ncu traffic record's staleness check."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from swiglu_ar_tts_b200.chain import DecodeChain  # noqa: E402
from swiglu_ar_tts_b200.inputs import ChainShape  # noqa: E402


def test_decode_step_algorithmic_bytes():
    """Per decode step: 28 x (B x 81,932 + 8,192) bytes (two add+norms, M-RoPE
    with 12 B of positions per row, SwiGLU, four gamma reads)."""
    for batch, want in ((5, 11_699_856), (256, 587_517_952)):
        shape = ChainShape(batch=batch)
        from swiglu_ar_tts_b200.inputs import decode_chain_inputs

        c = DecodeChain(shape, device="cpu", host_inputs=decode_chain_inputs(shape))
        assert c.bytes_per_step() == want
        assert c.launches_per_step == 112


def test_prefill_algorithmic_bytes():
    b = bench.step_bytes()
    assert b["rmsnorm"] == (2 * 64 * 1024 + 1024) * 4 == 528_384
    assert b["add_rmsnorm"] == (4 * 4096 * 2048 + 2048) * 2 == 67_112_960
    assert b["swiglu"] == 3 * 8192 * 6144 * 2 == 301_989_888
    assert b["mrope_qk"] == 2 * 4096 * 24 * 128 * 2 + 3 * 4096 * 4 == 50_380_800
    assert (b["decode_b5"], b["decode_b256"]) == (11_699_856, 587_517_952)
    assert sum(b.values()) == 1_019_229_840
    assert tuple(b) == bench.STEP_CONFIGS == bench.Step.OPS


def test_cpu_baseline_report_on_a_small_step(monkeypatch):
    """The CPU-baseline record: plain and row-parallel builds of the oracle,
    per-configuration times, host core count and CPU model (run here on a
    reduced step whose configurations are cut to a few rows)."""
    class Tiny(bench.OracleStep):
        def __init__(self):
            from swiglu_ar_tts_b200 import inputs
            f64 = lambda t: t.double().numpy()  # noqa: E731
            self.rn = {k: f64(v) for k, v in inputs.rmsnorm_inputs(4, 64, "f32", 0).items()}
            self.an = {k: f64(v) for k, v in inputs.add_rmsnorm_inputs(4, 64, "bf16", 0).items()}
            self.sw = {k: f64(v) for k, v in inputs.swiglu_inputs(4, 64, "bf16", 0).items()}
            mr = inputs.mrope_inputs(8)
            self.pos = mr["pos"].numpy()
            self.mr = {k: f64(v) for k, v in mr.items() if k != "pos"}
            shape = ChainShape(batch=2, layers=2)
            c = inputs.decode_chain_inputs(shape)
            chain = (f64(c["residual"]), {k: [f64(t) for t in v] for k, v in c.items() if k != "residual"})
            self.chains = {"decode_b5": chain, "decode_b256": chain}
            self.bytes = {k: 1000 for k in bench.STEP_CONFIGS}
            self.sample = "tiny"

    rep = bench.cpu_baseline_report(Tiny())
    assert rep["kind"] == "oracle" and rep["cores"] == 1 and rep["single"]["threads"] == 1
    assert rep["omp"]["threads"] >= 1 and rep["nproc"] >= 1 and rep["cpu_model"]
    assert set(rep["per_config_ms"]) == set(bench.STEP_CONFIGS)
    assert set(rep["omp"]["per_config_ms"]) == set(bench.STEP_CONFIGS)
    assert rep["value"] == rep["single"]["value"] > 0


def _rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local = [3.0, 5.0][rank]  # rank 1 is slower
    m = bench.reduce_max(local, dist, torch.device("cpu"))
    v = bench.aggregate_value(world, 1_000_000_000, 10, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, v))


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29517
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in res:
        assert m == 5.0  # both ranks see the slowest rank's time
        assert v == pytest.approx(2 * 1e9 * 10 / 5e-3 / 1e9)


def test_reference_arm_other_ranks_print_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reduce_max_without_group_is_identity():
    assert bench.reduce_max(2.5) == 2.5


@pytest.mark.parametrize("kernel", ["swiglu_vec_kernel", "norm_rows_kernel"])
def test_traffic_record_tracks_kernel_source(kernel):
    """The recorded traffic is DRAM reads plus bytes written into L2, reported
    only while the kernel's sources are the ones captured."""
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[kernel]
    got = bench.ncu_traffic(kernel, tuple(rec["sources"]))
    if rec["source_digest"] == bench.source_digest(*rec["sources"]):
        assert got == rec["traffic_bytes_per_launch"]
        assert got >= rec["dram_bytes_per_launch"]  # includes the writes still in L2
    else:  # the kernel changed since the capture: the bench must report null
        assert got is None
    assert bench.ncu_traffic("no_such_kernel", tuple(rec["sources"])) is None


def test_hbm_peak_source():
    peak, kind = bench.measured_hbm_peak()
    assert kind in ("measured", "fallback") and peak > 1000


@pytest.mark.parametrize("norm", ["rms", "layer"])
def test_decode_calls_group_by_operator(norm):
    """The bench's attribution groups a step's 112 launches as 56 norms, 28
    M-RoPE, 28 SwiGLU (CPU buffers: only the grouping is exercised)."""
    from swiglu_ar_tts_b200.inputs import decode_chain_inputs

    shape = ChainShape(batch=5)
    c = DecodeChain(shape, device="cpu", host_inputs=decode_chain_inputs(shape), norm=norm)
    groups = bench.group_decode_calls(c)
    norm_op = "add_layernorm" if norm == "layer" else "add_rmsnorm"
    assert {k: len(v) for k, v in groups.items()} == {norm_op: 56, "mrope_qk": 28, "swiglu": 28}
    assert all(bench.KERNEL_OF[k] for k in groups)


def test_e2e_pipeline_covers_every_operator_once():
    """The end-to-end pipeline copies in, runs and copies out every operator of
    the step exactly once, whatever order it takes them in."""
    names = [name for _, name in bench.Step.E2E_GROUPS]
    assert sorted(names) == sorted(bench.Step.OPS)
    groups = [g for g, _ in bench.Step.E2E_GROUPS]
    assert len(set(groups)) == len(groups)


def test_source_digest_ignores_comments_but_not_code(tmp_path):
    """The traffic records stay valid across comment edits and lapse on any
    change to the code they were measured with."""
    f = tmp_path / "k.cu"
    f.write_text("// kernel\n__global__ void k(int* p) { p[0] = 1; }  // store one\n")
    d0 = bench.source_digest(str(f))
    f.write_text("// the kernel, reworded\n\n__global__ void k(int* p) { p[0] = 1; }\n")
    assert bench.source_digest(str(f)) == d0
    f.write_text("// kernel\n__global__ void k(int* p) { p[0] = 2; }  // store one\n")
    assert bench.source_digest(str(f)) != d0
