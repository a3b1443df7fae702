"""Host-side checks of the C ABI: the library loads, exports every declared
entry point, and rejects bad arguments before touching the device (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_api():
    names = declared_functions()
    for must in ("attn_plan_create", "attn_select", "attn_forward", "attn_layer"):
        assert must in names


def test_library_exports_every_declared_symbol():
    from block_sparse_attention_reorder_b200 import bsattn
    lib = ctypes.CDLL(bsattn.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(bsattn.EXPORTED)


def test_status_strings():
    from block_sparse_attention_reorder_b200 import bsattn
    for code in range(7):
        assert bsattn.attn_status_string(code) == bsattn.STATUS[code]


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), 2),                     # unsupported head_dim
    (dict(tile=(3, 4, 6)), 2),                  # tile volume 72: above 64, not a multiple of 64
    (dict(tile=(2, 3, 32)), 2),                 # 64-row runs are not boxes (3 h rows of 32)
    (dict(tile=(8, 1, 24)), 2),                 # 24-token frames do not divide 64
    (dict(tile=(1, 1, 2048)), 2),               # a side above 1024
    (dict(T=0), 1),                             # empty grid
    (dict(B=0), 1),
    (dict(k=0), 1),                             # top-k needs k >= 1
    (dict(k=33), 1),                            # k > N (N = 32)
    (dict(rule="topp", k=2, p=0.0), 1),         # p outside (0, 1]
    (dict(rule="topp", k=2, p=1.5), 1),
    (dict(rule="topp", k=-1, p=0.5), 1),
    (dict(rule="window", win=(-1, 0, 0)), 1),
    (dict(rule=7), 1),
    (dict(T=4 * 32, H=4 * 8, W=4 * 9, k=8), 2),  # N = 2304 > 2048 for top-k
])
def test_plan_rejects_bad_arguments_before_any_device_call(kw, code):
    from block_sparse_attention_reorder_b200 import bsattn
    args = dict(B=1, heads=2, head_dim=64, T=8, H=16, W=16, rule="topk", k=8)
    args.update(kw)
    with pytest.raises(bsattn.BsattnError) as e:
        bsattn.Plan(**args)
    assert e.value.code == code


def test_null_plan_and_null_pointers_are_invalid():
    from block_sparse_attention_reorder_b200 import bsattn
    lib = bsattn._lib
    assert lib.attn_plan_create(None, None, None) == 1
    assert lib.attn_reorder(None, None, None, None, None) == 1
    assert lib.attn_forward(None, None, None, None, None, None, None, None, None, None, None, 0,
                            None) == 1
    assert lib.attn_layer(None, None, None, None, None, None, None, None, None, 0, None) == 1
    assert lib.attn_check_device_status(None, None) == 1
    assert lib.attn_backward(None, None, None, None, None, None, None, None, None, None, None, None, None, 0,
                             None) == 1
    assert lib.attn_plan_info(None, None) == 1
    lib.attn_plan_destroy(None)  # no-op


_GRID = dict(B=1, heads=2, head_dim=64, T=8, H=16, W=16)


@pytest.mark.parametrize("entries", [
    [],                                                              # no entry
    [(1, dict(rule="topk", k=8))],                                   # does not start at step 0
    [(0, dict(rule="topk", k=8)), (0, dict(rule="topk", k=4))],      # first steps not increasing
    [(0, dict(rule="topk", k=8)), (5, dict(rule="topk", k=4)), (3, dict(rule="topk", k=2))],
    [(0, dict(rule="topk", k=8))] + [(i, dict(rule="topk", k=8)) for i in range(1, 65)],  # > 64
])
def test_schedule_rejects_bad_entries_before_any_device_call(entries):
    from block_sparse_attention_reorder_b200 import bsattn
    with pytest.raises(bsattn.BsattnError) as e:
        bsattn.Schedule(**_GRID, entries=entries)
    assert e.value.code == 1


def test_schedule_rejects_entries_over_different_tensors():
    from block_sparse_attention_reorder_b200 import bsattn
    arr = (bsattn.ScheduleEntry * 2)()
    for i, T in enumerate((8, 12)):  # a different grid in the second entry
        arr[i].first_step = 10 * i
        arr[i].desc = bsattn.Desc(1, 2, 64, T, 16, 16, 4, 4, 4, 0.0, 0)
        arr[i].rule = bsattn.Rule(0, 8, 0.0, 0, 0, 0)
    h = ctypes.c_void_p()
    assert bsattn._lib.attn_schedule_create(arr, 2, ctypes.byref(h)) == 1
    assert not h.value


def test_null_schedule_calls_are_invalid():
    from block_sparse_attention_reorder_b200 import bsattn
    lib = bsattn._lib
    assert lib.attn_schedule_create(None, 1, None) == 1
    assert lib.attn_schedule_plan(None, 0, None) == 1
    assert lib.attn_schedule_workspace_bytes(None, None) == 1
    assert lib.attn_schedule_layer(None, 0, None, None, None, None, None, None, None, None, 0,
                                   None) == 1
    lib.attn_schedule_destroy(None)  # no-op
