"""bench.bench_configs's control flow on CPU: CUDA events, the L2 flush and
the library calls are stand-ins, so this checks the leg's wiring -- inputs
per config, the FLOP count, per-step and per-kernel times, the graph branch,
the single-rank rule for it and the error capture -- not any GPU number."""
import argparse
import types

import torch

import bench


class _Ev:
    def __init__(self, enable_timing=False):
        pass

    def record(self, stream=None):
        pass

    def elapsed_time(self, other):
        return 0.5


class _FakeCuda:
    Event = _Ev

    @staticmethod
    def current_stream():
        return None

    @staticmethod
    def synchronize():
        pass

    @staticmethod
    def empty_cache():
        pass


class _TorchProxy:
    """torch, except that CUDA is faked and device buffers are small host ones."""
    cuda = _FakeCuda

    def __getattr__(self, name):
        return getattr(torch, name)

    @staticmethod
    def empty(*size, dtype=None, device=None):
        return torch.empty(16, dtype=dtype)


def _fake_api(calls, fail_graph=False, fail_cfg4=False):
    def fwd_gate(q, k, v, g, scale, return_workspace=False, **kw):
        calls.append(("fwd_gate", tuple(q.shape), kw.get("cu_seqlens") is not None))
        return q, q[..., 0], g.float(), torch.empty(1)

    def bwd(dO, q, k, v, P, o, lse, scale, **kw):
        calls.append(("bwd", kw.get("want_dsink", False), kw.get("fwd_workspace") is not None))
        if fail_cfg4 and kw.get("cu_seqlens") is not None:
            raise RuntimeError("planted")
        return q, k, v, q, None, None

    def prefix(g, cu=None):
        calls.append(("prefix", cu is not None))
        return g.float()

    def fwd(q, k, v, P, scale, **kw):
        calls.append(("fwd", kw.get("window_size")))
        return q, q[..., 0]

    class Graph:
        def __init__(self, *a, **kw):
            if fail_graph:
                raise RuntimeError("capture refused")
            self.graph = types.SimpleNamespace(replay=lambda: calls.append(("replay",)))

    return types.SimpleNamespace(
        wall_attn_fwd_gate=fwd_gate, wall_attn_bwd=bwd, prefix_cumsum=prefix, wall_attn_fwd=fwd,
        WallAttnStepGraph=Graph, timing_enable=lambda on=True: None,
        timing_read=lambda: {"fwd_tc": (10, 1.0), "bwd_keyblock": (10, 2.0), "decode": (0, 0.0)})


def _run(monkeypatch, world=1, **fail):
    calls = []
    import channel_decay_softmax_b200 as pkg
    monkeypatch.setattr(pkg, "api", _fake_api(calls, **fail), raising=False)
    monkeypatch.setitem(__import__("sys").modules, "channel_decay_softmax_b200.api",
                        _fake_api(calls, **fail))
    monkeypatch.setattr(bench, "torch", _TorchProxy())
    real = bench.I.training_inputs
    monkeypatch.setattr(bench.I, "training_inputs",
                        lambda s, device="cpu", lengths=None: real(
                            bench.I.spec(s.n_seq and 4 or 2, seed=s.seed,
                                         **({"len_lo": 8, "len_hi": 16} if s.n_seq else
                                            {"T": 16})), "cpu", lengths))
    monkeypatch.setattr(bench, "max_over_ranks", lambda x, w: x)
    out = bench.bench_configs(argparse.Namespace(steps=10, warmup=3), world, 0)
    return out, calls


def test_both_configs_timed_per_step_kernel_and_graph(monkeypatch):
    out, calls = _run(monkeypatch)
    c2, c4 = out["config2"], out["config4"]
    for c in (c2, c4):
        assert "error" not in c, c
        assert c["ms_per_step"] == 0.5 and c["kernel_ms_per_step"] == 3.0 / 10
        assert abs(c["tflops"] - c["fwd_bwd_flop"] / 0.5e-3 / 1e12) < 1e-9
        assert abs(c["kernel_tflops"] - c["fwd_bwd_flop"] / 0.3e-3 / 1e12) < 1e-9
    assert c2["graph_ms_per_step"] == 0.5 and "graph_tflops" in c2
    assert "graph_ms_per_step" not in c4
    assert "packed sequences" in c4["workload"] and "window 1024" in c4["workload"]
    # both through the gate call, the backward reusing its workspace; config 4
    # (packed sequences, with a sink) asks for dsink
    assert ("bwd", False, True) in calls and ("bwd", True, True) in calls
    assert any(c[0] == "fwd_gate" and c[2] for c in calls)  # packed sequences
    assert not any(c[0] in ("prefix", "fwd") for c in calls)
    for name, row in c4["stage_ms_per_step"].items():
        assert row > 0, name
    assert any(c[0] == "replay" for c in calls)


def test_graph_only_in_single_rank_runs_and_errors_are_reported(monkeypatch):
    out, _ = _run(monkeypatch, world=2)
    assert out["config2"]["graph"] == "single-rank runs only"
    out, _ = _run(monkeypatch, fail_graph=True)
    assert out["config2"]["graph_error"].startswith("RuntimeError")
    assert "tflops" in out["config2"]
    out, _ = _run(monkeypatch, fail_cfg4=True)
    assert out["config4"] == {"error": "RuntimeError: planted"}
    assert "tflops" in out["config2"]
