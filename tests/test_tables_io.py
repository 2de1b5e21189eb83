"""Tables files (ace_tables_save / ace_tables_info / ace_tables_load): the
offline tables of a table build kept on disk and reloaded ([ACE] "Practical
Implications": the tables depend only on the frozen weights, so one build
serves every later run).  Host code, no GPU.  A reload must give the same
bits; a torn, corrupted, truncated or foreign file, and a file of another
shape, must be refused without touching the caller's arrays."""
import os

import pytest
import torch

from token_dynamic_expert_b200 import ace


def _tables(L=3, E=16, seed=0):
    g = torch.Generator().manual_seed(seed)
    a_gsp = torch.rand(L, E, generator=g) + 0.5
    a_rcr = torch.rand(L, E, generator=g) + 0.5
    return a_gsp, a_rcr, torch.maximum(a_gsp, a_rcr), torch.rand(L, E, 3, generator=g) * 4


def test_round_trip_is_bit_exact(tmp_path):
    a_gsp, a_rcr, amax, sigma = _tables()
    p = str(tmp_path / "t.acetbl")
    ace.ace_tables_save(p, a_gsp, a_rcr, amax, sigma)
    assert not os.path.exists(p + ".tmp")
    assert ace.ace_tables_info(p) == (3, 16, True)
    g, r, m, s = ace.ace_tables_load(p, with_sigma=True)
    for a, b in ((g, a_gsp), (r, a_rcr), (m, amax), (s, sigma)):
        assert torch.equal(a, b)
    # without sigma
    p2 = str(tmp_path / "t2.acetbl")
    ace.ace_tables_save(p2, a_gsp, a_rcr, amax)
    assert ace.ace_tables_info(p2) == (3, 16, False)
    g, r, m = ace.ace_tables_load(p2)
    assert torch.equal(m, amax)
    with pytest.raises(ace.AceError) as e:
        ace.ace_tables_load(p2, with_sigma=True)
    assert e.value.code == ace.ACE_ERR_INVALID_ARG
    # the file is the documented layout: 32-byte header, then the arrays
    assert os.path.getsize(p) == 32 + 4 * 3 * 16 * (3 + 3)
    with open(p, "rb") as f:
        head = f.read(32)
    assert head[:8] == b"ACETBL\x00\x01"
    assert int.from_bytes(head[12:16], "little") == 3 and int.from_bytes(head[16:20], "little") == 16


def _load_code(p, L=3, E=16):
    out = [torch.full((L, E), 7.0) for _ in range(3)]
    code = ace.lib().ace_tables_load(os.fsencode(p), L, E, *(ace._ptr(t) for t in out), None)
    return code, out


@pytest.mark.parametrize("damage", ["flip", "truncate", "extend", "magic", "missing"])
def test_damaged_files_are_refused(tmp_path, damage):
    a_gsp, a_rcr, amax, sigma = _tables()
    p = str(tmp_path / "t.acetbl")
    ace.ace_tables_save(p, a_gsp, a_rcr, amax, sigma)
    data = bytearray(open(p, "rb").read())
    if damage == "flip":
        data[100] ^= 0x01
    elif damage == "truncate":
        data = data[:-4]
    elif damage == "extend":
        data += b"\x00"
    elif damage == "magic":
        data[0] = ord("X")
    if damage == "missing":
        os.remove(p)
    else:
        open(p, "wb").write(bytes(data))
    code, out = _load_code(p)
    assert code == ace.ACE_ERR_IO
    assert all(torch.equal(t, torch.full((3, 16), 7.0)) for t in out)  # untouched


def test_shape_mismatch_and_bad_arguments(tmp_path):
    a_gsp, a_rcr, amax, _ = _tables()
    p = str(tmp_path / "t.acetbl")
    ace.ace_tables_save(p, a_gsp, a_rcr, amax)
    code, out = _load_code(p, L=3, E=8)
    assert code == ace.ACE_ERR_INVALID_ARG
    assert all(torch.equal(t, torch.full((3, 8), 7.0)) for t in out)
    lib = ace.lib()
    assert lib.ace_tables_save(os.fsencode(p), 0, 16, ace._ptr(a_gsp), ace._ptr(a_rcr),
                               ace._ptr(amax), None) == ace.ACE_ERR_INVALID_ARG
    assert lib.ace_tables_save(os.fsencode(p), 3, 16, None, ace._ptr(a_rcr), ace._ptr(amax),
                               None) == ace.ACE_ERR_INVALID_ARG
    # an unwritable path
    bad = str(tmp_path / "no_such_dir" / "t.acetbl")
    assert lib.ace_tables_save(os.fsencode(bad), 3, 16, ace._ptr(a_gsp), ace._ptr(a_rcr),
                               ace._ptr(amax), None) == ace.ACE_ERR_IO
    assert ace.ace_status_str(ace.ACE_ERR_IO) == "ACE_ERR_IO"


def test_save_replaces_an_existing_file(tmp_path):
    p = str(tmp_path / "t.acetbl")
    a = _tables(seed=1)
    b = _tables(L=2, E=32, seed=2)
    ace.ace_tables_save(p, *a[:3])
    ace.ace_tables_save(p, *b)
    assert ace.ace_tables_info(p) == (2, 32, True)
    assert torch.equal(ace.ace_tables_load(p)[2], b[2])
