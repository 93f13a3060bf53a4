"""The relation the forward's sequence split links its segments by, checked in
fp64 on the oracle alone (no device code).

The recurrence ("TorchMamba" README, "Math notes", M3 SISO) is linear in the
state and its rotation angles add, so for a sequence cut at token s the state
after the last token satisfies

    h_T = exp(sum of logdecay over tokens s..T-1) h_{s-1}
          + R(phi_{s-1}) hloc,

where hloc is the state the tail builds from a zero start with its own angle
counted from zero (the carry-in token s-1 entering unrotated), and R rotates
each pair (2i, 2i+1) of the state's rows by phi_{s-1, i}.  The device splits
sequences this way (its segment pass writes hloc in the frame of the segment's
last token, which is the same rotation applied in two steps); a mistake in the
decay sum, the carry-in token or the rotation's sign breaks these equalities."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs


def rot_pairs(h, phi):
    """R(phi) on the row pairs of h (..., N, P): (c re - s im, s re + c im)."""
    c, s = np.cos(phi)[..., None], np.sin(phi)[..., None]
    re, im = h[..., 0::2, :], h[..., 1::2, :]
    out = np.empty_like(h)
    out[..., 0::2, :] = c * re - s * im
    out[..., 1::2, :] = s * re + c * im
    return out


def cached_inputs(seed=31, L=200):
    w = WORKLOADS["tiny"].with_(batch=2, seqlen=L, nheads=4, ngroups=2, headdim=4, dstate=8,
                                seed=seed)
    inp = make_inputs(w)
    g = torch.Generator().manual_seed(seed + 1)
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    inp["h0"] = torch.randn(b, H, N, P, generator=g) * 0.3
    inp["angle0"] = torch.rand(b, H, N // 2, generator=g) * 6 - 3
    inp["xprev0"] = torch.randn(b, H, P, generator=g)
    inp["bprev0"] = torch.randn(b, G, N, generator=g) / N ** 0.5
    return inp


def part(inp, sl):
    keys = ("X", "logdecay", "beta", "gamma", "B", "C", "theta")
    return {k: (None if inp[k] is None else inp[k][:, sl].contiguous()) for k in keys}


@pytest.mark.parametrize("cut", [1, 63, 100, 199])
def test_tail_from_zero_start_links_to_the_one_pass_state(cut):
    inp = cached_inputs()
    full = oracle.oracle_fwd(**inp)
    head = oracle.oracle_fwd(**part(inp, slice(0, cut)), D=inp["D"], h0=inp["h0"],
                             angle0=inp["angle0"], xprev0=inp["xprev0"], bprev0=inp["bprev0"])
    # the tail from a zero state and a zero angle; its carry-in token is token cut-1, unrotated
    tail = oracle.oracle_fwd(**part(inp, slice(cut, None)), D=inp["D"],
                             xprev0=inp["X"][:, cut - 1].double(),
                             bprev0=inp["B"][:, cut - 1].double())
    decay = np.exp(inp["logdecay"][:, cut:].double().numpy().sum(axis=1))  # (b, H)
    linked = decay[..., None, None] * head["hT"] + rot_pairs(tail["hT"], head["angleT"])
    np.testing.assert_allclose(linked, full["hT"], rtol=1e-9, atol=1e-12)
    # the angles add: the tail's own angle sum on top of the head's
    d = tail["angleT"] + head["angleT"] - full["angleT"]
    assert np.max(np.abs((d + np.pi) % (2 * np.pi) - np.pi)) < 1e-9


def test_three_segments_chain():
    """Two cuts, linked in order from the first segment's state, as the combine
    step does for segments 1 .. S-1."""
    inp = cached_inputs(seed=37, L=240)
    full = oracle.oracle_fwd(**inp)
    cuts = [0, 80, 170, 240]
    h = inp["h0"].double().numpy()
    phi = inp["angle0"].double().numpy()
    for k in range(3):
        lo, hi = cuts[k], cuts[k + 1]
        if k == 0:
            seg = oracle.oracle_fwd(**part(inp, slice(lo, hi)), D=inp["D"], xprev0=inp["xprev0"],
                                    bprev0=inp["bprev0"])
        else:
            seg = oracle.oracle_fwd(**part(inp, slice(lo, hi)), D=inp["D"],
                                    xprev0=inp["X"][:, lo - 1].double(),
                                    bprev0=inp["B"][:, lo - 1].double())
        decay = np.exp(inp["logdecay"][:, lo:hi].double().numpy().sum(axis=1))
        h = decay[..., None, None] * h + rot_pairs(seg["hT"], phi)
        phi = phi + seg["angleT"]
    np.testing.assert_allclose(h, full["hT"], rtol=1e-9, atol=1e-12)


def test_wrong_carry_in_breaks_the_link():
    """Differ-guard: the tail started without its carry-in token (its beta term
    dropped) does not link to the one-pass state."""
    inp = cached_inputs(seed=41)
    cut = 197  # near the end, so that the decay leaves the beta term visible
    full = oracle.oracle_fwd(**inp)
    head = oracle.oracle_fwd(**part(inp, slice(0, cut)), D=inp["D"], h0=inp["h0"],
                             angle0=inp["angle0"], xprev0=inp["xprev0"], bprev0=inp["bprev0"])
    tail = oracle.oracle_fwd(**part(inp, slice(cut, None)), D=inp["D"])
    decay = np.exp(inp["logdecay"][:, cut:].double().numpy().sum(axis=1))
    linked = decay[..., None, None] * head["hT"] + rot_pairs(tail["hT"], head["angleT"])
    rms = np.sqrt(np.mean(full["hT"] ** 2))
    assert np.max(np.abs(linked - full["hT"])) > 1e-3 * rms
