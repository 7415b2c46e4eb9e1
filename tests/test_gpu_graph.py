"""Training steps replayed as CUDA graphs equal eager steps bit for bit.

With graph=True the trainer runs the first step of each kind eagerly, records
the next one (kernels, layer uploads, the events that order them) as a CUDA
graph through lsq_stream_capture_begin / _end, and replays it from then on.
The replay must compute exactly what the eager steps compute: the same loss
curve, LoRA gradients, logits and adapter weights, the same upload counts and
the same number of kernel launches.  Covered:

* streamed layers through two slots, a streamed lm_head, a resident run;
* the 3B shape at 512 tokens (tiles shared out by stream-K across clusters,
  whose flags a replay reuses) and the 8B shape at 2048 tokens (a stream-K
  tail), both cut to a few full-width layers;
* graph steps mixed with eager steps and with DPO steps in one run (the
  scheduler's events recorded inside a capture are recorded again at the next
  eager use).
"""
import dataclasses

import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu


def _cut(shape, n_layers):
    return dataclasses.replace(shape, name=f"{shape.name}-{n_layers}l", n_layers=n_layers)


def _drive(tr, shape, B, Sq, plan):
    """Run the plan's steps ("sft", "dpo", "eager-sft"); returns the losses, the last step's
    gradients and logits, the adapter weights and the kernel launches issued."""
    from nf4_layer_streamed_blockwise_b200 import lib as L
    losses = []
    n0 = L.LAUNCHES[0]
    for t, kind in enumerate(plan):
        tr.set_ids(S.tokens(shape, B, Sq, step=t).cuda())
        if kind.startswith("eager"):
            tr.timeline = []            # instrumented steps run eagerly
        if kind.endswith("dpo"):
            tr.forward_backward_dpo(0.1)
        else:
            tr.forward_backward()
        tr.timeline = None
        losses.append(tr.loss_dev.item())
        tr.optimizer_step()
    torch.cuda.synchronize()
    return losses, tr.lora.grad.clone(), tr.logits.clone(), tr.lora.master.clone(), L.LAUNCHES[0] - n0


def _pair(shape, B, Sq, plan, **kw):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    side = torch.cuda.Stream()
    out = []
    with torch.cuda.stream(side):
        for graph in (False, True):
            tr = StreamedLoraTrainer(shape, B, Sq, init="device", graph=graph, **kw)
            res = _drive(tr, shape, B, Sq, plan)
            out.append((res, tr.stats(), tr.head_stats(), set(tr._graphs)))
            tr.close()
    return out


def _same(eager, graph):
    (el, eg, elog, ew, en), est, ehs, _ = eager
    (gl, gg, glog, gw, gn), gst, ghs, kinds = graph
    assert el == gl, (el, gl)
    assert torch.equal(eg, gg)
    assert torch.equal(elog, glog)
    assert torch.equal(ew, gw)
    assert est == gst and ehs == ghs, (est, gst, ehs, ghs)
    assert en == gn, (en, gn)
    return kinds


@pytest.mark.parametrize("case", ["tiny-2slots", "tiny-untied-head-host", "tiny-resident", "qwen3b-4l-512",
                                  "llama8b-2l-2048"])
def test_graph_replay_equals_eager_bitwise(lsq, case):
    shape, B, Sq, kw = {
        "tiny-2slots": (S.TINY, 2, 96, dict(n_slots=2)),
        "tiny-untied-head-host": (S.TINY_UNTIED, 2, 128, dict(n_slots=2, head="host", head_chunk=256)),
        "tiny-resident": (S.TINY, 2, 96, dict(n_slots=None)),
        "qwen3b-4l-512": (_cut(S.QWEN3B, 4), 1, 512, dict(n_slots=2)),
        "llama8b-2l-2048": (_cut(S.LLAMA8B, 2), 4, 512, dict(n_slots=2)),
    }[case]
    eager, graph = _pair(shape, B, Sq, ["sft"] * 5, **kw)
    assert _same(eager, graph) == {"sft"}


def test_graph_steps_mixed_with_eager_and_dpo(lsq):
    plan = ["sft", "sft", "sft", "eager-sft", "sft", "dpo", "dpo", "dpo", "sft", "eager-dpo", "dpo", "sft"]
    eager, graph = _pair(S.TINY, 2, 96, plan, n_slots=3)
    assert _same(eager, graph) == {"sft", ("dpo", 0.1)}


def test_graph_needs_a_side_stream(lsq):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    with pytest.raises(ValueError):
        StreamedLoraTrainer(S.TINY, 1, 64, n_slots=2, init="device", graph=True)   # default stream


def test_capture_refuses_a_stream_not_capturing(lsq):
    from nf4_layer_streamed_blockwise_b200 import lib as L
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        tr = StreamedLoraTrainer(S.TINY, 1, 64, n_slots=2, init="device")
        with pytest.raises(L.LsqError) as e:
            L.lsq_stream_capture_begin(tr.sched)
        assert L.STATUS[e.value.status] == "LSQ_ESTATE"
        with pytest.raises(L.LsqError) as e:
            L.lsq_stream_capture_end(tr.sched)
        assert L.STATUS[e.value.status] == "LSQ_ESTATE"
        tr.close()
