"""How dfw_decode_lanes_seq splits a sequence of scopes into launches (host
only, no GPU): one persistent launch per run of consecutive scopes that share
a CTA shape, at most DFW_SEQ_MAX_SCOPES scopes per run.  The query checks the
scopes as the call does and dereferences none of their buffers, so host
tensors stand in for the device ones here."""
import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads

MAX_SCOPES = 40


def _host_scope(u: np.ndarray) -> dfw.DeviceLanes:
    enc = dfw.encode(u)
    pl = dfw.plan_lanes(enc)
    return dfw.DeviceLanes(enc.stream, enc.mant, pl.lut, pl.chunk_bits, pl.group_start, enc.table, pl.info)


@pytest.fixture(scope="module")
def kinds():
    gauss = np.concatenate([workloads.as_u16_numpy(t) for t in
                            workloads.generate_block(workloads.scaled(workloads.c5()[1], 70_000))])
    rng = np.random.default_rng(3)
    single = ((rng.integers(0, 2, 5000) << 15) | (119 << 7) | rng.integers(0, 128, 5000)).astype(np.uint16)
    # uniform 16-bit patterns: all 256 exponents with 8-bit codes, a closed
    # form (codes read in place, no table); with exponent 0 folded into 1,
    # 255 exponents and codes of 7 and 8 bits: 2 KB group spans, too big for
    # the 1024-thread CTA
    closed = workloads.as_u16_numpy(workloads.generate_block(workloads.c4("c", 70_000))[0])
    wide = closed.copy()
    e = (wide >> 7) & 0xFF
    wide[e == 0] |= np.uint16(1 << 7)
    empty = _host_scope(np.zeros(0, np.uint16))
    empty.mant = torch.zeros(16, dtype=torch.uint8)  # a scope's raw-byte pointer may not be null, even when empty
    return {"gauss": _host_scope(gauss), "single": _host_scope(single), "wide": _host_scope(wide),
            "closed": _host_scope(closed), "empty": empty}


def test_model_sized_sequence_is_one_launch(kinds):
    g = kinds["gauss"]
    assert dfw.decode_lanes_seq_launches([g] * 34) == 1
    assert dfw.decode_lanes_seq_launches([g] * MAX_SCOPES) == 1
    assert dfw.decode_lanes_seq_launches([g] * (MAX_SCOPES + 1)) == 2
    assert dfw.decode_lanes_seq_launches([g] * (3 * MAX_SCOPES)) == 3
    assert dfw.decode_lanes_seq_launches([]) == 0


def test_runs_break_where_the_cta_shape_changes(kinds):
    g, w = kinds["gauss"], kinds["wide"]
    assert w.info.max_group_bytes > 2 * g.info.max_group_bytes
    assert dfw.decode_lanes_seq_launches([g, g, w, g, g]) == 3
    assert dfw.decode_lanes_seq_launches([w, w, w]) == 1


def test_fills_and_empty_scopes_take_no_launch_of_their_own(kinds):
    g, s, e, w, c = kinds["gauss"], kinds["single"], kinds["empty"], kinds["wide"], kinds["closed"]
    assert dfw.decode_lanes_seq_launches([g, s, g, e, g]) == 1
    assert dfw.decode_lanes_seq_launches([w, s, w]) == 1
    assert dfw.decode_lanes_seq_launches([s]) == 1
    assert dfw.decode_lanes_seq_launches([e, e]) == 0
    # a closed form needs no table or stream slot either
    assert c.table.n_symbols == 256 and all(c.table.len[x] == 8 for x in range(256))
    assert w.table.n_symbols == 255
    assert dfw.decode_lanes_seq_launches([g, c, g, c, g]) == 1
    assert dfw.decode_lanes_seq_launches([w, c, w]) == 1
    assert dfw.decode_lanes_seq_launches([c]) == 1


def test_bad_scope_is_refused(kinds):
    g = kinds["gauss"]
    bad = dfw.DeviceLanes(g.stream, g.mant, g.lut, g.chunk_bits, g.group_start, g.table,
                          dfw.LanesInfo.from_buffer_copy(bytes(g.info)))
    bad.info.n_chunks += 1
    with pytest.raises(dfw.DfwError) as ei:
        dfw.decode_lanes_seq_launches([g, bad])
    assert ei.value.status == dfw.EINVAL
