"""Which per-call options bench.py's step passes to the binding, on CPU with a recording stand-in
for the binding: seq_lens_ready on every single-launch call (one token, several tokens, the
prologue folded in), and never on the three-launch path, whose attention entry point would
refuse it."""
from dataclasses import replace
from types import SimpleNamespace

import torch

import bench
from load_balanced_split_step_b200 import workloads as W


class Recorder:
    """Stands in for the binding module: records each call's name and keyword arguments."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args, **kw):
            self.calls.append((name, kw))
            if name in ("plan", "plan_static"):
                return SimpleNamespace(workspace=None)
            if name == "partial_buffers":
                return None, None
            return None
        return call

    def kwargs_of(self, name):
        return [kw for n, kw in self.calls if n == name]


def _dc(spec):
    B, pages = spec.batch, 4
    return {"seq_lens": torch.full((B,), 8, dtype=torch.int32), "block_table": torch.zeros((B, pages), dtype=torch.int32),
            "q": torch.zeros((B, spec.num_heads, spec.head_dim), dtype=torch.bfloat16), "k_pages": None,
            "v_pages": None, "k_scale": None, "v_scale": None, "qkv": None, "q_norm_w": None, "k_norm_w": None}


def _run(spec, **kw):
    rec = Recorder()
    step = bench.Step(rec, spec, _dc(spec), 4, spec.tile_len, **kw)
    rec.calls.clear()
    step()
    return rec


def test_single_launch_one_token_sets_it():
    rec = _run(W.config_spec("tiny"), fused=True)
    (kw,) = rec.kwargs_of("decode_step_fused")
    assert kw["seq_lens_ready"] is True


def test_single_launch_several_tokens_sets_it():
    rec = _run(replace(W.config_spec("tiny"), q_len=3), fused=True)
    (kw,) = rec.kwargs_of("decode_step_multi")
    assert kw["seq_lens_ready"] is True


def test_folded_prologue_sets_it():
    spec = W.custom_spec((8, 9), 8, 2, 64, 16, 32, prologue=True)
    rec = _run(spec, folded=True)
    (kw,) = rec.kwargs_of("decode_step_prologue")
    assert kw["seq_lens_ready"] is True


def test_three_launches_do_not():
    rec = _run(W.config_spec("tiny"), fused=False)
    names = [n for n, _ in rec.calls]
    assert names == ["plan", "attention", "merge"]
    assert all("seq_lens_ready" not in kw for _, kw in rec.calls)
