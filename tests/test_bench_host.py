"""Host-side logic of bench.py that needs no GPU: the FLOP conventions, the digest
that ties committed ncu counters to the kernel code, and the reference arm's line."""
import importlib.util
import json
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_flop_conventions(bench):
    # forward 2*B*H*N^2*d causal (4* non-causal), backward credited 2.5x the forward
    assert bench.flops_fwd() == 2.0 * 2 * 16 * 4096 ** 2 * 128 == pytest.approx(137.44e9, rel=1e-3)
    assert bench.flops_fwd(causal=False) == 2 * bench.flops_fwd()
    assert bench.flops_bwd() == 2.5 * bench.flops_fwd()


def test_backward_phase_tables(bench):
    # each kernel's tensor-core FLOPs in units of the forward's two products: the single
    # pass does the method's five backward products once (S^T, dP^T, dV, dQ, dK = 2.5
    # forwards); the two-pass backward recomputes S and dP in its dQ kernel (4 + 3 = 7
    # products = 3.5 forwards).  Phase numbers as the C ABI's attn_bwd_phase.
    single = [(ph, k, m) for _, ph, k, m in bench.BWD_PHASES]
    det = [(ph, k, m) for _, ph, k, m in bench.BWD_PHASES_DET]
    assert [p for p, _, _ in single] == [3, 4, 5] and [p for p, _, _ in det] == [0, 1, 2]
    assert sum(m for _, _, m in single if m) == 2.5 and sum(m for _, _, m in det if m) == 3.5
    assert {k for _, k, m in single + det if m is None} == {"attn_bwd_pre_kernel", "attn_bwd_dq_convert_kernel"}
    # the tensor-core kernels' names are the record keys of their ncu reports at the bench's
    # instantiations, which the roofline looks up for its traffic
    for _, k, m in single + det:
        if m is not None:
            args = "128, 0, 0" if "fused" in k else "128, 0"
            assert bench.ncu_kernel_key(f"void attn::{k}<{args}>(CUtensorMap_st, P)") == k


def _copy_sources(tmp_path):
    dst = tmp_path / "exact_attention_123_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "exact_attention_123_b200", "csrc"), dst,
                    ignore=shutil.ignore_patterns("*.o", "*.so"))
    return dst


def test_digest_ignores_comments_but_not_code(bench, tmp_path, monkeypatch):
    base = bench.source_digest()
    src = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    assert bench.source_digest() == base
    f = src / "attn_fwd_sm100.cu"
    text = f.read_text(encoding="utf-8")
    f.write_text("// a new comment line\n/* and a block\n   comment */\n" + text.replace("\n", "\n\n", 3),
                 encoding="utf-8")
    assert bench.source_digest() == base
    f.write_text(text.replace("kRescaleThreshold = 8.0f", "kRescaleThreshold = 9.0f"), encoding="utf-8")
    assert bench.source_digest() != base


def test_recorded_counters_only_for_matching_code(bench, tmp_path, monkeypatch):
    _copy_sources(tmp_path)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    good = bench.source_digest()
    rec = {"k_match": {"source_digest": good, "dram_bytes_per_launch": 123, "tensor_pipe_active_pct": 50.0},
           "k_stale": {"source_digest": "0000000000000000", "dram_bytes_per_launch": 456}}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("k_match") == 123
    assert bench.recorded_traffic("k_stale") is None
    assert bench.recorded_traffic("absent") is None
    got = bench.recorded_ncu()
    assert set(got) == {"k_match"} and got["k_match"]["tensor_pipe_active_pct"] == 50.0


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOPS" and line["value"] > 0
    assert line["higher_is_better"] is True and line["steps"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_ncu_report_rows(bench):
    # the raw-page CSV of `ncu -i REPORT --page raw --csv`: a header row, a units row,
    # then one row per captured launch
    head = ["ID", "Kernel Name", "gpu__time_duration.sum", "dram__bytes_read.sum", "dram__bytes_write.sum",
            "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed",
            "launch__shared_mem_per_block_dynamic", "l1tex__data_bank_conflicts_pipe_lsu_mem_shared_op_st.sum"]
    units = ["", "", "usecond", "Mbyte", "Kbyte", "%", "Kbyte", ""]
    rows = [["0", "void attn::attn_bwd_dkdv_sm100_kernel<128, 0>(CUtensorMap_st, BwdParams)", "200", "150.5",
             "2,048", "51.5", "216.184", "7"],
            ["1", "void attn::attn_fwd_sm100_kernel<128, 0, 1>(CUtensorMap_st, FwdParams)", "100", "50", "5",
             "27.5", "214.2", "0"]]
    text = "\n".join(",".join(f'"{c}"' for c in r) for r in [head, units] + rows)
    got = bench.ncu_rows(text)
    assert [e["kernel"] for e in got] == ["attn_bwd_dkdv_sm100_kernel", "attn_fwd_sm100_kernel<128, 0, 1>"]
    e = got[0]
    assert e["dram_bytes_per_launch"] == 150_500_000 + 2_048_000
    assert e["hbm_gbs"] == pytest.approx(152_548_000 / 200e-6 / 1e9)
    assert e["tensor_pipe_active_pct"] == 51.5 and e["smem_per_cta_kb"] == 216.184
    assert e["smem_bank_conflicts_st"] == 7
    assert bench.ncu_kernel_key("void attn::attn_fwd_sm100_kernel<64, 1, 0>(X)") == "attn_fwd_sm100_kernel<64, 1, 0>"


def test_launch_plan_honours_gpus(bench):
    # one plain process and --gpus 1: run here
    assert bench.launch_plan(1, {}) == ("run", None)
    # under a launcher whose world size matches: run here
    assert bench.launch_plan(4, {"WORLD_SIZE": "4"}) == ("run", None)
    # one plain process asked for N > 1 GPUs: relaunch as N ranks, one per GPU, on 127.0.0.1
    plan, argv = bench.launch_plan(2, {})
    assert plan == "spawn"
    assert "torch.distributed.run" in argv and "--nproc-per-node=2" in argv and "--master-addr=127.0.0.1" in argv
    assert argv[-1 - len(sys.argv[1:])].endswith("bench.py")
    # a launcher with another world size: refuse instead of printing the wrong n_gpus
    plan, why = bench.launch_plan(2, {"WORLD_SIZE": "1"})
    assert plan == "error" and "WORLD_SIZE=1" in why
    assert bench.launch_plan(0, {})[0] == "error"


def test_gpus_mismatch_exits_nonzero():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1"],
                       capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode != 0
    assert "WORLD_SIZE=1" in json.loads(r.stdout.strip().splitlines()[-1])["error"]
