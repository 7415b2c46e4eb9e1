"""The layer-streaming slot policy, checked on CPU through lsq_stream_simulate
(the same decision code lsq_stream_step executes with CUDA events).

Ordering invariants over the emitted actions:
* compute waits for a layer only while its slot holds that layer;
* a slot is overwritten only after its previous occupant, if compute used it,
  was released (the copy stream waits on that release);
* the layer in use is never overwritten;
* steady-state uploads per training step = 2 (L - n_slots): the last n_slots
  layers of the forward and the first ones of the backward are reused.
"""
import pytest

RELEASE, UPLOAD, WAIT = 1, 2, 3


def _train_steps(L, steps):
    out = []
    for _ in range(steps):
        out += [(l, +1) for l in range(L)]
        out += [(l, -1) for l in reversed(range(L))]
    return out


def _check(L, S, steps, acts):
    holds = {}            # slot -> layer
    used = {}             # slot -> occupant was waited on since its upload
    released = {}         # slot -> occupant released since its last use
    in_use = None
    waits = [a for a in acts if a[0] == WAIT]
    assert [(l) for _, l, _ in waits] == [l for l, _ in steps]
    for kind, layer, slot in acts:
        assert 0 <= slot < S
        if kind == UPLOAD:
            if holds.get(slot) is not None and used.get(slot):
                assert released.get(slot), f"slot {slot} overwritten before release of layer {holds[slot]}"
            assert not (in_use is not None and holds.get(slot) == in_use), "layer in use was evicted"
            for s2, l2 in list(holds.items()):      # a layer lives in one slot at a time
                if l2 == layer and s2 != slot:
                    del holds[s2]
            holds[slot], used[slot], released[slot] = layer, False, False
        elif kind == WAIT:
            assert holds.get(slot) == layer, f"compute on layer {layer} but slot {slot} holds {holds.get(slot)}"
            used[slot], released[slot] = True, False
            in_use = layer
        elif kind == RELEASE:
            assert holds.get(slot) == layer
            released[slot] = True
        else:
            raise AssertionError(kind)


@pytest.mark.parametrize("L", [3, 30, 32])
@pytest.mark.parametrize("S", [2, 3, 4, 8])
def test_policy_invariants_and_upload_count(L, S):
    from nf4_layer_streamed_blockwise_b200 import lib
    if S > L:
        pytest.skip("more slots than layers")
    steps = _train_steps(L, 4)
    acts = lib.lsq_stream_simulate(L, S, steps)
    _check(L, S, steps, acts)
    # steady state: uploads during the last training step
    one = 2 * L
    acts_last = lib.lsq_stream_simulate(L, S, steps[:-one])
    up_before = sum(1 for a in acts_last if a[0] == UPLOAD)
    up_all = sum(1 for a in acts if a[0] == UPLOAD)
    assert up_all - up_before == 2 * (L - S)


def test_resident_uploads_each_layer_once():
    from nf4_layer_streamed_blockwise_b200 import lib
    L = 30
    steps = _train_steps(L, 3)
    acts = lib.lsq_stream_simulate(L, L, steps)
    _check(L, L, steps, acts)
    ups = [a for a in acts if a[0] == UPLOAD]
    assert sorted(l for _, l, _ in ups) == list(range(L))


def test_random_walk_keeps_invariants():
    import random
    from nf4_layer_streamed_blockwise_b200 import lib
    rng = random.Random(0)
    for S in (2, 3, 5, 8):
        L = 17
        steps, l, d = [], 0, 1
        for _ in range(400):
            if rng.random() < 0.1:
                d = -d
            elif rng.random() < 0.05:
                l = rng.randrange(L)
            steps.append((l, d))
            l = min(max(l + d, 0), L - 1)
        _check(L, S, steps, lib.lsq_stream_simulate(L, S, steps))


def test_bad_arguments():
    from nf4_layer_streamed_blockwise_b200 import lib
    with pytest.raises(lib.LsqError):
        lib.lsq_stream_simulate(4, 9, [(0, 1)])
    with pytest.raises(lib.LsqError):
        lib.lsq_stream_simulate(4, 2, [(4, 1)])
    with pytest.raises(lib.LsqError):
        lib.lsq_stream_simulate(4, 2, [(0, 0)])


@pytest.mark.parametrize("name", ["tiny", "smollm2-135m", "llama-3.1-8b", "dense-32b"])
def test_record_layout_double_quant(name):
    """The double-quantised record: smaller than the fp32 one by 3 bytes per block
    (less the params), every piece aligned and disjoint, the expanded fp32
    arrays after the record inside the slot, and the byte count bench.py reports."""
    import bench
    import synthetic as S
    from nf4_layer_streamed_blockwise_b200.trainer import RecordLayout
    sh = S.SHAPES[name]
    f, q = RecordLayout.of(sh, "fp32"), RecordLayout.of(sh, "dq8")
    assert f.slot_bytes == f.nbytes and f.dq is None
    assert q.nbytes < f.nbytes and q.slot_bytes > q.nbytes
    assert abs(q.nbytes - bench.record_bytes(sh, "dq8")) < 64 * 256       # alignment padding only
    spans = [(q.codes[n], q.codes[n] + a * b // 2) for n, (a, b) in sh.linear_shapes().items()]
    spans += [(c8, c8 + nb) for c8, _, nb in q.dq.values()]
    spans += [(pp, pp + 8 * ((nb + 255) // 256)) for _, pp, nb in q.dq.values()]
    spans += [(q.ln1, q.ln1 + 2 * sh.d), (q.ln2, q.ln2 + 2 * sh.d)]
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:])) and spans[-1][1] <= q.nbytes
    assert all(s % 256 == 0 for s, _ in spans)
    outs = sorted((o, o + 4 * nb) for _, _, o, nb in q.expand_items())
    assert outs[0][0] >= q.nbytes and outs[-1][1] <= q.slot_bytes
    assert all(a[1] <= b[0] for a, b in zip(outs, outs[1:]))
    if name == "llama-3.1-8b":
        assert abs(q.nbytes / 1e6 - 112.5) < 0.2 and abs(f.nbytes / 1e6 - 122.7) < 0.1
    with pytest.raises(ValueError):
        RecordLayout.of(sh, "int8")


def test_store_sizes_match_the_pages():
    """The whole pinned store with double-quantised records comes to the sizes
    the pages print for the 8B and 3B runs (tests/golden/ram_store_sizes.json);
    with fp32 absmax it is about 9% larger."""
    import json
    import os
    import synthetic as S
    from nf4_layer_streamed_blockwise_b200.trainer import RecordLayout
    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "ram_store_sizes.json")))
    for name, gb in gold["values"].items():
        sh = S.SHAPES[name]
        dq = sh.n_layers * RecordLayout.of(sh, "dq8").nbytes / 1e9
        f32 = sh.n_layers * RecordLayout.of(sh, "fp32").nbytes / 1e9
        assert round(dq, 2) == gb, (name, dq)
        assert 1.08 < f32 / dq < 1.10, (name, f32, dq)
