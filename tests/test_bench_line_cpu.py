"""The bench's stdout line on CPU: built from a full record of the shape run_ours makes.

The line must hold every key of the bench contract, keep the whole decode object (the
second half of the metric) at its end, and stay short enough that a consumer keeping
only the last ~3 KB of output still sees all of it.
"""
import json

import bench


def _full_record():
    rl = {"bound": "alu", "unit": "Gexp/s", "achieved": 2464.866200253, "peak": 4653.12,
          "frac": 0.52972332547, "traffic": 654278144.0, "algorithmic_bytes": 673816576,
          "hbm_GBps": 1099.94921641, "hbm_frac": 0.16800299615, "peak_note": "x" * 90,
          "kernel_ms": 0.61258880496}
    dec_rl = {"bound": "hbm", "unit": "GB/s", "achieved": 4758.1234567, "peak": 6547.2,
              "frac": 0.72674123, "algorithmic_bytes": 178601984, "peak_kind": "measured",
              "traffic": None}
    return {
        "metric": bench.METRIC, "value": 136208068821.32565, "unit": "elems/s", "n_gpus": 1,
        "steps": 2000, "warmup": 20, "ms_per_step": 0.6158671855926514,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "io_dtype": "bf16", "data": "synthetic", "impl": "ours",
        "config": {"workload": "w" * 90, "batch": 4, "dim": 5120, "dstate": 16, "seqlen": 4096,
                   "l2": "no flush", "parallelism": "replicas x1 (independent batches per GPU)"},
        "roofline": rl,
        "cpu_baseline": {"value": 49666300.37, "unit": "elems/s", "cores": 16, "kind": "oracle",
                         "cpu_model": "Intel(R) Xeon(R) Processor",
                         "single_thread_value": 6947542.58,
                         "sample": "20480 of 20480 channels x full L=4096 (fp64, sequential per "
                                   "channel, 16 OpenMP threads), 1.7 s; single thread: 2429 "
                                   "channels, 2.5 s"},
        "e2e": {"value": 8576569995.460849, "unit": "elems/s", "h2d_bytes_per_step": 504365056,
                "d2h_bytes_per_step": 167772160, "ms_per_step": 9.780842463175455, "steps": 12,
                "pipeline": "p" * 60},
        "gpu_launches": 2000,
        "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 13,
                   "power_w_median": 471.0},
        "decode": {"metric": "decode state-updates/s", "unit": "(b,d) lane updates/s",
                   "value": 34952533333.3, "steps_per_s": 26666.67,
                   "ms_per_token_l2_flushed": 0.0375, "ms_per_token_back_to_back": 0.0328,
                   "workload": "d" * 80, "roofline": dec_rl, "gpu_launches": 2005},
        "backward": {"value": 2.49e10, "ms_per_call": 3.37, "roofline": {"frac": 0.193},
                     "train_step": {"ms_per_step": 3.54, "roofline": {"frac": 0.275}},
                     "cpu_baseline": {"sample": "s" * 90}},
        "exact_zoh": {"ms_per_call": 0.962, "roofline": {"frac": 0.337},
                      "backward": {"ms_per_call": 4.1, "roofline": {"frac": 0.16}},
                      "decode": {"ms_per_token_l2_flushed": 0.0412, "roofline": {"frac": 0.66}}},
        "conv1d": {"ms_per_call": 0.0575, "roofline": {"frac": 0.89},
                   "backward": {"ms_per_call": 0.0912, "roofline": {"frac": 0.84}},
                   "decode": {"ms_per_token_l2_flushed": 0.0124, "roofline": {"frac": 0.26}}},
        "lshard": None,
        "workloads": {"m130m": {"ms": 0.218, "value": 1.156e11, "frac": 0.447},
                      "million": {"ms": 25.5, "value": 8.43e10, "frac": 0.326},
                      "gpu_launches": 150},
        "pipe_probes": {"note": "n" * 200},
    }


def test_compact_line_keeps_contract_keys_and_fits_the_tail():
    out = bench.compact_line(_full_record())
    text = json.dumps(out)
    assert len(text) < 2600, len(text)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in out, k
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in out["roofline"], k
    for k in ("value", "unit", "cores", "kind", "sample"):
        assert k in out["cpu_baseline"], k
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in out["e2e"], k
    assert list(out)[-1] == "decode"
    assert out["decode"]["roofline"]["frac"] == 0.72674
    assert out["value"] == 1.3621e11
    # the decode object is whole inside the last 1 KB of the line
    assert text[-1000:].find('"decode"') >= 0
