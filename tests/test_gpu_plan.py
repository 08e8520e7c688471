"""GPU: the staged decode's automatic partition plan, read back from the workspace.

With num_splits = 0 the plan kernel lays the contexts end to end and cuts them into
one equal token range per SM, snapping each cut inside a sequence to a 16-token
tile of that sequence; a range's pieces (its parts of consecutive sequences) are
one CTA's units.  Read back after a decode call, the plan must cover every token of
every sequence exactly once, in pieces that start on a tile, number each sequence's
pieces 0 .. ns[b] - 1 within the partial-result slots the workspace holds, and give
no CTA more than the range (plus one tile of snapping) of tokens."""
import numpy as np
import pytest
import torch

from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.CONFIGS


def _up256(x):
    return (x + 255) // 256 * 256


def _read_plan(ws, B, P):
    """(ns[B], units[n], cta_off[P + 1], range) from the workspace layout: a 256-byte
    header (unit counter, unit count, range, ...), ns at byte 256, the unit list
    (int4 b, c, t0, t1; room for B + P), then the per-CTA unit offsets."""
    head = ws[:16].view(torch.int32).cpu().numpy()
    n_units, rng = int(head[1]), int(head[2])
    off_units = 256 + _up256(4 * B)
    off_cta = off_units + _up256(16 * (B + P))
    ns = ws[256:256 + 4 * B].view(torch.int32).cpu().numpy()
    units = ws[off_units:off_units + 16 * n_units].view(torch.int32).cpu().numpy().reshape(-1, 4)
    cta = ws[off_cta:off_cta + 4 * (P + 1)].view(torch.int32).cpu().numpy()
    return ns, units, cta, rng


@pytest.mark.parametrize("key", ["c2m", "c3m", "c4m", "c5m", "ragged"])
def test_balanced_plan_covers_every_token_once(key):
    cases = {
        "c2m": W.scaled(C["c2"], key="pc2", layers=1, batch=32, old_lens=(1024,) * 32,
                        score=False),
        "c3m": W.scaled(C["c3"], key="pc3", layers=1, batch=9, old_len_range=(1, 3000)),
        "c4m": W.scaled(C["c4"], key="pc4", batch=2, old_lens=(20000, 300)),
        "c5m": W.scaled(C["c5"], key="pc5", batch=12, old_lens=(4096,) * 12),
        "ragged": W.scaled(C["c3"], key="prg", layers=1, batch=6,
                           old_lens=(0, 15, 16, 17, 1000, 0), append=False),
    }
    wl = W.generate(cases[key], "cpu")
    cfg = wl.cfg
    ref = oracle_step(wl, 0, range(cfg.batch))
    dev = Device(wl)
    if cfg.int8:
        dev.fill_int8_history(0)
    dev.step(0)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert_attention_close(dev.out[0], ref["out"], key)
    P = torch.cuda.get_device_properties(0).multi_processor_count
    B = cfg.batch
    ns, units, cta, rng = _read_plan(dev.ws, B, P)
    lens = wl.ctx_lens
    S = pk.pa_decode_plan(B, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size, wl.max_blocks)[0]
    assert len(units) <= B + P
    assert cta[0] == 0 and (np.diff(cta) >= 0).all() and cta[-1] == len(units)
    assert rng % 16 == 0 and rng >= 128
    seen = {b: [] for b in range(B)}
    for i in range(P):
        tok = 0
        for b, c, t0, t1 in units[cta[i]:cta[i + 1]]:
            assert 0 <= b < B and 0 <= c < ns[b] <= S
            assert 0 <= t0 < t1 <= lens[b] and t0 % 16 == 0
            seen[b].append((c, t0, t1))
            tok += t1 - t0
        assert tok <= rng + 16, (i, tok, rng)
    for b in range(B):
        if lens[b] == 0:
            assert ns[b] == 0 and not seen[b]
            continue
        pieces = sorted(seen[b])
        assert [p[0] for p in pieces] == list(range(ns[b]))
        assert pieces[0][1] == 0 and pieces[-1][2] == lens[b]
        assert all(e0 == a1 for (_, _, e0), (_, a1, _) in zip(pieces, pieces[1:]))
