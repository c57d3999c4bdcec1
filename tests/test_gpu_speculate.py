"""Self-speculative greedy decode on the GPU path against the fp64 oracle
("CLI Reference", speculate: --draft-loops / --verify-loops / --draft-ahead,
temperature 0).  The oracle's speculative_lane gives the tokens (with greedy
choices, those of a plain decode at the verify depth) and the number of verify
rounds; the GPU must emit the same tokens wherever the oracle's verify-depth
logits have a top-1/top-2 margin above 1e-3, and, up to the first near-tie,
run the same rounds."""
import numpy as np
import pytest

import synthetic as S
from oracle import decode as D
from oracle import model as M

from gpu_helpers import MARGIN, gpu_model, oracle_weights, status_clean

pytestmark = pytest.mark.gpu


def _first_near_tie(ref_plain):
    for t in range(len(ref_plain.tokens)):
        if M.top2_margin(ref_plain.logits[t]) <= MARGIN:
            return t
    return len(ref_plain.tokens)


@pytest.mark.parametrize("name,L_draft,L_verify,ahead", [("tiny", 2, 8, 4), ("tiny", 1, 4, 3), ("tiny", 4, 4, 5),
                                                         ("m407", 2, 8, 4)])
def test_speculate_matches_oracle(name, L_draft, L_verify, ahead):
    sh = S.SHAPES[name]
    W = oracle_weights(name)
    T, n_new = 12, 10
    P = S.prompts(2, T, sh.vocab, seed=121)
    m = gpu_model(name, None, max_lanes=max(2, ahead), max_seq=T + n_new + 1, L_max=8,
                  max_prefill_tokens=max(T, ahead))
    for i in range(2):
        ref_tok, ref_rounds = D.speculative_lane(W, P[i], L_draft, L_verify, n_new, ahead)
        plain = D.generate_lane(W, P[i], L_verify, n_new)
        assert np.array_equal(ref_tok, plain.tokens)
        m.prefill(i, P[i], L_verify)
        tok, rounds = m.speculate(i, n_new, L_draft, L_verify, ahead)
        status_clean(m)
        stop = _first_near_tie(plain)
        assert tok[:stop].tolist() == ref_tok[:stop].tolist(), (i, tok, ref_tok)
        if stop == n_new:
            assert rounds == ref_rounds, (i, rounds, ref_rounds)
        if L_draft == L_verify:  # every draft is accepted
            assert rounds == -(-(n_new - 1) // ahead)


def test_speculate_refusals():
    from dynamic_depth_b200 import TlError
    m = gpu_model("tiny", None, max_lanes=4, max_seq=32, L_max=8, max_prefill_tokens=16)
    P = S.prompts(1, 8, 512, seed=122)
    m.prefill(0, P[0], 4)
    with pytest.raises(TlError) as e:
        m.speculate(0, 5, 2, 8, 4)   # verify deeper than the lane's cache
    assert e.value.status == -4
    with pytest.raises(TlError) as e:
        m.speculate(1, 5, 2, 4, 4)   # lane never prefilled
    assert e.value.status == -3
    # a second call continues from where the first left the lane: its first token is the first call's last
    tok, _ = m.speculate(0, 5, 2, 4, 4)
    tok2, _ = m.speculate(0, 4, 2, 4, 4)
    status_clean(m)
    W = oracle_weights("tiny")
    plain = D.generate_lane(W, P[0], 4, 8)
    stop = _first_near_tie(plain)
    assert tok.tolist()[:stop] == plain.tokens[:5].tolist()[:stop]
    assert (tok.tolist() + tok2.tolist()[1:])[:stop] == plain.tokens.tolist()[:stop]
