"""Invariants of the oracle's multi-step decode loop (CPU only)."""

import numpy as np

import synth
from oracle import decode, stage


def _run(gain, noise, seeds, S=16, V=4096, d=128):
    W = synth.bf16_bits(synth.weights(V, d))
    return decode.decode_batch(W, W, seeds, decode.stub_hidden_fn(W, seeds, S, gain, noise), V,
                               max_steps=S, record=True), W


def test_stop_invariants_and_commit():
    seeds = [0, 1, 2]
    r, _ = _run(300.0, 0.1, seeds)
    S = 16
    assert (r["stop_step"] < S).any()                # the early-stop branch is exercised
    for c in range(3):
        s_stop = int(r["stop_step"][c])
        assert 1 <= s_stop <= S
        if s_stop < S:
            assert s_stop >= 3                       # three identical argmax vectors needed
        last = r["trace"][s_stop - 1]["canvases"][c]
        assert np.array_equal(r["committed"][c], last["argmax"])
        if s_stop < S:
            assert last["mean_H"] < 0.005 and last["stable"] >= 2
        # no earlier step satisfied both conditions
        for rec in r["trace"][:s_stop - 1]:
            cc = rec["canvases"][c]
            assert not (cc["mean_H"] < 0.005 and cc["stable"] >= 2)
        # a stopped canvas is never touched again
        for rec in r["trace"][s_stop:]:
            assert c not in rec["canvases"]


def test_tokens_follow_accept_rule():
    seeds = [4]
    r, _ = _run(150.0, 0.1, seeds)
    for rec in r["trace"]:
        cc = rec["canvases"][0]
        acc = cc["H"] <= 0.1
        assert np.array_equal(cc["accept"].astype(bool), acc)
        assert np.array_equal(cc["tokens"][acc], cc["argmax"][acc])
        ren = stage.renoise_tokens(4, rec["s"], 0, 4096)
        assert np.array_equal(cc["tokens"][~acc], ren[~acc])


def test_literal_gain_never_accepts():
    # the unscaled stub keeps every entropy near ln V: nothing is accepted, no early stop
    r, _ = _run(1.0, 0.1, [0], S=6)
    assert r["stop_step"][0] == 6
    for rec in r["trace"]:
        assert rec["canvases"][0]["accept"].sum() == 0
