"""Host logic the GPU stream tests rely on, checked on the CPU.

first_divergent_cycle decides which cycle's decision margin may excuse a
divergence between a GPU stream and the oracle's: it must return -1 for a
stream equal to the oracle's (up to the first N tokens) and otherwise the
index of the first cycle whose length or tokens differ, never a later one.
"""
import oracle
import synth
from gpu_helpers import first_divergent_cycle

N = 20


def _reference(n_tokens=N, K=4):
    m = oracle.Model(synth.make_weights(synth.TINY, 0))
    return m.generate(synth.make_prompt(synth.TINY, 16, 0), K, n_tokens, 0.0, 0, "orthrus")


def _cycles(ref):
    out, pos = [], 0
    for n in ref["n_per_cycle"]:
        n = int(n)
        out.append((n, [int(x) for x in ref["tokens"][pos:pos + n]]))
        pos += n
    return out


def test_equal_stream_has_no_divergence():
    ref = _reference()
    cyc = _cycles(ref)
    assert len(cyc) == ref["cycles"] >= 2
    assert first_divergent_cycle(cyc, ref, N) == -1


def test_token_change_is_found_at_its_cycle():
    ref = _reference()
    for c in range(len(_cycles(ref))):
        cyc = _cycles(ref)
        n, toks = cyc[c]
        if not toks:
            continue
        toks = list(toks)
        toks[-1] = (toks[-1] + 1) % synth.TINY.vocab
        cyc[c] = (n, toks)
        assert first_divergent_cycle(cyc, ref, N) == c


def test_length_change_is_found_at_its_cycle():
    ref = _reference()
    cyc = _cycles(ref)
    c = len(cyc) // 2
    n, toks = cyc[c]
    cyc[c] = (n + 1, toks + [0])                     # one more token accepted than the oracle did
    assert first_divergent_cycle(cyc, ref, N) == c
    # and a later difference does not hide it
    cyc[-1] = (cyc[-1][0], [(t + 1) % synth.TINY.vocab for t in cyc[-1][1]])
    assert first_divergent_cycle(cyc, ref, N) == c


def test_tokens_past_n_are_not_compared():
    ref = _reference()
    cyc = _cycles(ref)
    # the oracle stopped at N; anything a GPU run emitted after N is ignored
    cyc.append((3, [1, 2, 3]))
    assert first_divergent_cycle(cyc, ref, N) == -1
    # a last cycle that runs past N is compared on its first tokens only
    # (13 tokens end inside a two-token cycle of this stream)
    ref13 = _reference(13)
    cyc = _cycles(ref13)
    pos = sum(n for n, _ in cyc[:-1])
    n, toks = cyc[-1]
    kept = 13 - pos
    assert 0 < kept < n and len(toks) == kept          # the oracle keeps only the tokens up to N
    cyc[-1] = (n, toks + [7] * (n - kept))             # a GPU cycle emits all n; the rest is free
    assert first_divergent_cycle(cyc, ref13, 13) == -1
    cyc[-1] = (n, [(toks[0] + 1) % synth.TINY.vocab] + toks[1:] + [7] * (n - kept))
    assert first_divergent_cycle(cyc, ref13, 13) == len(cyc) - 1


def test_fewer_accepted_or_more_cycles_is_a_divergence():
    ref = _reference()
    cyc = _cycles(ref)
    c = next(i for i, (n, _) in enumerate(cyc) if n > 1)
    cyc[c] = (1, cyc[c][1][:1])                        # the GPU accepted fewer at cycle c
    assert first_divergent_cycle(cyc, ref, N) == c
    short = dict(ref, cycles=1)                        # an oracle run that ended after one cycle
    assert first_divergent_cycle(_cycles(ref), short, 10 ** 6) == 1
