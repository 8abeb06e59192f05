"""Host-side summary of a concurrent kernel timeline (profile_timeline):
per-kernel means, the step span and one layer's window, on a synthetic trace."""

from looped_transformer_latent_b200 import profile_timeline as pt


def _ev(name, ts, dur, stream, grid, cat="kernel"):
    return {"ph": "X", "cat": cat, "name": name, "ts": ts, "dur": dur,
            "args": {"stream": stream, "grid": grid}}


def test_report_means_span_and_layer_window(capsys):
    events = []
    # two replays of a two-layer step: per layer a map and a read on two streams
    for r in range(2):
        for layer in range(2):
            t = 100.0 * (2 * r + layer)
            events.append(_ev("void lla::(anonymous namespace)::tc_gemm<0, 32, 1>(x)", t, 10.0, 7, [4, 64, 1]))
            events.append(_ev("void lla::(anonymous namespace)::absorb_split_tc(y)", t + 12.0, 50.0 + r, 8, [4, 32, 1]))
    events.append({"ph": "i", "cat": "kernel", "name": "marker", "ts": 0.0})   # not a duration event
    pt.report(events, replays=2, layers=2, layer=1)
    out = capsys.readouterr().out
    lines = out.splitlines()
    assert lines[1].split()[:2] == ["absorb_split_tc", "[4,"]          # largest total first
    assert "50.5" in lines[1] and " 4 " in lines[1]                    # 4 launches, mean 50.5 us
    assert "tc_gemm<0, 32, 1>" in lines[2] and "10.0" in lines[2]
    assert "step: 181.5 us" in out                                     # (300 + 12 + 51 - 0) / 2
    window = [ln for ln in lines if ln.strip().startswith("100.0") or ln.strip().startswith("112.0")]
    assert len(window) == 2                                            # layer 1 of the first replay


def test_empty_trace(capsys):
    pt.summarise([], replays=1, layer_window=None)
    assert "no GPU activity" in capsys.readouterr().out
