"""The C-ABI library loads, exports every symbol include/*.h declares, and
rejects bad arguments on the host before any CUDA call (runs without a GPU)."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("pkv.h", "pkv_pages.h")]


@pytest.fixture(scope="module")
def pkv():
    from paged_kv_flight_b200 import build
    build.build()
    from paged_kv_flight_b200 import pkv as mod
    return mod


def _declared():
    text = "".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z_]+)\s*\(", text)))


def test_header_declarations_are_all_exported(pkv):
    names = _declared()
    assert set(names) == set(pkv.EXPORTS)
    for n in names:
        assert hasattr(pkv.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", pkv._LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) <= exported


def test_config_struct_layout_matches_header(pkv):
    # ints, enum, then a double on an 8-byte boundary, then three ints
    assert C.sizeof(pkv.pkv_config) == 48
    assert pkv.pkv_config.rope_base.offset == 24


def _cfg(pkv, **kw):
    base = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=32, kv_dtype=0,
                rope_base=5e5, max_batch=64, max_blocks_per_seq=129, num_pages=5000)
    base.update(kw)
    return pkv.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(num_q_heads=30), 1),                      # Hq % Hkv != 0
    (dict(num_kv_heads=0), 1),
    (dict(head_dim=96), 2),
    (dict(head_dim=-1), 1),
    (dict(page_size=8), 2),
    (dict(page_size=0), 1),
    (dict(num_q_heads=128, num_kv_heads=8), 2),     # G = 16
    (dict(kv_dtype=7), 1),
    (dict(rope_base=1.0), 1),
    (dict(rope_base=float("nan")), 1),
    (dict(max_batch=0), 1),
    (dict(max_batch=100000), 2),
    (dict(num_pages=0), 1),
    (dict(max_blocks_per_seq=0), 1),
])
def test_create_rejects_bad_configs_on_the_host(pkv, kw, status):
    st, ctx = pkv.pkv_create(_cfg(pkv, **kw), check=False)
    assert st == status and ctx is None


def test_null_context_and_status_strings(pkv):
    assert pkv.lib.pkv_rope_append(None, None, None, None, None, None, None, None, None, 1, None, 1, None) == 1
    assert pkv.lib.pkv_decode_attn(None, None, None, None, None, None, None, 1, None, 1, None, None) == 1
    assert pkv.lib.pkv_set_workers(None, 3) == 1
    assert pkv.lib.pkv_set_tail_chunks(None, 3) == 1
    assert pkv.lib.pkv_destroy(None) == 0
    assert pkv.lib.pkv_workspace_bytes(None) == 0
    for s in range(7):
        assert pkv.pkv_status_str(s) and pkv.pkv_status_str(s) != "unknown status"
    assert pkv.pkv_status_str(99) == "unknown status"


def test_table_sync_rejects_bad_sizes_without_touching_the_device():
    """Argument checks of pkv_table_sync run on the host before any launch."""
    import torch
    from paged_kv_flight_b200 import pkv
    t = torch.zeros(4, 8, dtype=torch.int32)
    up = torch.zeros(64, dtype=torch.int32)
    bt, ln = torch.zeros(4, 8, dtype=torch.int32), torch.zeros(4, dtype=torch.int32)
    call = lambda n, b, P: pkv.pkv_table_sync(up, n, b, t, bt, ln, P, stream=0, check=False)   # noqa: E731
    assert call(-1, 1, 16) == pkv.PKV_ERR_INVALID_ARG
    assert call(0, 5, 16) == pkv.PKV_ERR_INVALID_ARG      # batch above the table's rows
    assert call(0, 1, 0) == pkv.PKV_ERR_INVALID_ARG       # page size
    assert call(0, 0, 16) == pkv.PKV_OK                    # nothing to do
