"""The C-ABI boundary without a GPU: the library loads, exports every entry
point include/lq.h declares, validates configs and lays out workspaces.
No call here launches a kernel."""
import ctypes

import pytest

from recurrent_state_quantization_lq_b200 import lq


def test_exports_every_declared_symbol():
    names = lq.header_symbols()
    assert set(names) >= {"lq_workspace_bytes", "lq_workspace_layout", "lq_state_create",
                          "lq_prefill_state", "lq_decode_step", "lq_window_flush", "lq_window_fill",
                          "lq_device_status", "lq_state_destroy", "lq_last_error_string",
                          "lq_decode_step_active", "lq_window_flush_pending", "lq_prefill_sequences",
                          "lq_prefill_tokens", "lq_prefill_sequences_tokens", "lq_state_resume",
                          "lq_state_export"}
    L = lq.lib()
    for n in names:
        assert hasattr(L, n), n


@pytest.mark.parametrize("mode", ["window", "naive", "fp32"])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("d", [64, 128])
def test_layout_regions_disjoint_aligned(mode, gate, d):
    cfg = lq.make_config(3, 5, d, window=37, n_comp_rows=3, n_comp_cols=1, gate=gate, mode=mode)
    L = lq.workspace_layout(cfg)
    assert L.total_bytes == lq.workspace_bytes(cfg) > 0
    N = 15
    key_b = 4 if gate == "channel" else 2
    sizes = {"err": 256, "codes": N * d * d, "row_scale": N * d * 4, "col_smooth": N * d * 4,
             "comp_index": N * L.comp_index_stride * 4, "comp_row_vec": N * 3 * d * 4,
             "comp_col_vec": N * 1 * d * 4, "gate_sum": N * (d if gate == "channel" else 1) * 8,
             "buf_delta": N * 37 * d * 4, "buf_key": N * 37 * d * key_b,
             "buf_gate": N * L.window_pad * 4, "state_f32": N * d * d * 4}
    present = {
        "window": {"err", "codes", "row_scale", "col_smooth", "comp_index", "comp_row_vec", "comp_col_vec",
                   "gate_sum", "buf_delta", "buf_key"} | ({"buf_gate"} if gate == "scalar" else set()),
        "naive": {"err", "codes", "row_scale"},
        "fp32": {"err", "state_f32"},
    }[mode]
    spans = []
    for name, size in sizes.items():
        off = getattr(L, name)
        if name in present:
            assert off != lq.ABSENT and off % 256 == 0 and off + size <= L.total_bytes, name
            spans.append((off, off + size))
        else:
            assert off == lq.ABSENT, name
    spans.sort()
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0
    if mode == "window":
        assert L.comp_index_stride == 4 and L.window_pad == 40


@pytest.mark.parametrize("field,value", [("d_k", 96), ("d_v", 64), ("window", 0), ("window", 5000),
                                         ("n_comp_rows", 9), ("n_comp_cols", -1), ("gate", 2),
                                         ("mode", 3), ("smooth", 2), ("select", 2), ("in_dtype", 3),
                                         ("batch", 0), ("heads", 0)])
def test_invalid_configs_rejected(field, value):
    cfg = lq.make_config(2, 2, 128)
    setattr(cfg, field, value)
    assert lq.workspace_bytes(cfg) == 0
    assert lq.last_error() != ""
    L = lq.Layout()
    assert lq.lib().lq_workspace_layout(ctypes.byref(cfg), ctypes.byref(L)) == lq.LQ_ERR_INVALID_ARG


def test_create_checks_workspace_and_lifecycle():
    L = lq.lib()
    cfg = lq.make_config(2, 2, 64, window=8)
    need = lq.workspace_bytes(cfg)
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: create is host-only
    assert L.lq_state_create(ctypes.byref(cfg), None, need, ctypes.byref(h)) == lq.LQ_ERR_WORKSPACE
    assert L.lq_state_create(ctypes.byref(cfg), ctypes.c_void_p((1 << 20) + 16), need,
                             ctypes.byref(h)) == lq.LQ_ERR_WORKSPACE
    assert L.lq_state_create(ctypes.byref(cfg), fake, need - 1, ctypes.byref(h)) == lq.LQ_ERR_WORKSPACE
    assert "needs" in lq.last_error()
    assert L.lq_state_create(ctypes.byref(cfg), fake, need, ctypes.byref(h)) == lq.LQ_OK
    assert L.lq_window_fill(h) == 0
    # decode and flush before prefill are refused on the host, before any launch
    p = ctypes.c_void_p(1 << 21)
    assert L.lq_decode_step(h, p, p, p, p, p, p, None) == lq.LQ_ERR_STATE
    assert L.lq_window_flush(h, None) == lq.LQ_ERR_STATE
    # null and misaligned inputs
    assert L.lq_decode_step(h, None, p, p, p, p, p, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_decode_step(h, ctypes.c_void_p((1 << 21) + 8), p, p, p, p, p, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_state_destroy(h) == lq.LQ_OK
    assert L.lq_window_fill(None) == -1
    assert L.lq_state_destroy(None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_prefill_state(None, None, None) == lq.LQ_ERR_INVALID_ARG


def test_flush_is_noop_outside_windowed_mode():
    L = lq.lib()
    for mode in ("naive", "fp32"):
        cfg = lq.make_config(1, 1, 64, mode=mode)
        h = ctypes.c_void_p()
        assert L.lq_state_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), lq.workspace_bytes(cfg),
                                 ctypes.byref(h)) == lq.LQ_OK
        assert L.lq_window_flush(h, None) == lq.LQ_OK
        L.lq_state_destroy(h)


def test_ragged_layout_and_validation():
    cfg = lq.make_config(3, 5, 128, window=37, ragged=True)
    L = lq.workspace_layout(cfg)
    assert L.fill != lq.ABSENT and L.fill % 256 == 0
    assert L.fill + 15 * 4 <= L.total_bytes
    shared = lq.workspace_layout(lq.make_config(3, 5, 128, window=37))
    assert shared.fill == lq.ABSENT
    for mode in ("naive", "fp32"):
        assert lq.workspace_bytes(lq.make_config(3, 5, 128, mode=mode, ragged=True)) == 0
    bad = lq.make_config(3, 5, 128)
    bad.ragged = 2
    assert lq.workspace_bytes(bad) == 0


def test_ragged_entry_points_check_the_handle_kind():
    L = lq.lib()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: every call below returns before any launch
    shared, ragged = ctypes.c_void_p(), ctypes.c_void_p()
    cs = lq.make_config(2, 3, 64, window=8)
    cr = lq.make_config(2, 3, 64, window=8, ragged=True)
    assert L.lq_state_create(ctypes.byref(cs), fake, lq.workspace_bytes(cs), ctypes.byref(shared)) == lq.LQ_OK
    assert L.lq_state_create(ctypes.byref(cr), fake, lq.workspace_bytes(cr), ctypes.byref(ragged)) == lq.LQ_OK
    p = ctypes.c_void_p(1 << 21)
    # shared-phase handles refuse the ragged calls
    assert L.lq_decode_step_active(shared, p, p, p, p, p, None, p, None) == lq.LQ_ERR_STATE
    assert L.lq_prefill_sequences(shared, None, p, None) == lq.LQ_ERR_STATE
    assert L.lq_prefill_sequences_tokens(shared, None, p, p, p, p, p, 4, None, p, None, None) == lq.LQ_ERR_STATE
    # ragged handles: counts live on the device; order of calls is checked on the host
    assert L.lq_window_fill(ragged) == -1
    assert L.lq_window_fill(shared) == 0
    assert L.lq_prefill_sequences(ragged, None, p, None) == lq.LQ_ERR_STATE      # before lq_prefill_state
    assert L.lq_window_flush_pending(ragged, None) == lq.LQ_ERR_STATE            # before lq_prefill_state
    assert L.lq_prefill_sequences_tokens(ragged, None, p, p, p, p, p, 4, None, p, None, None) == lq.LQ_ERR_STATE
    assert L.lq_decode_step_active(ragged, p, p, p, p, p, None, p, None) == lq.LQ_ERR_STATE
    assert L.lq_state_destroy(shared) == lq.LQ_OK
    assert L.lq_state_destroy(ragged) == lq.LQ_OK


def test_prefill_tokens_validates_on_the_host():
    L = lq.lib()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: every call below returns before any launch
    h = ctypes.c_void_p()
    cfg = lq.make_config(2, 3, 64, window=8, gate="channel")
    assert L.lq_state_create(ctypes.byref(cfg), fake, lq.workspace_bytes(cfg), ctypes.byref(h)) == lq.LQ_OK
    p = ctypes.c_void_p(1 << 21)
    assert L.lq_prefill_tokens(h, None, p, p, p, p, p, -1, None, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_prefill_tokens(h, None, None, p, p, p, p, 4, None, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_prefill_tokens(h, None, p, p, p, None, p, 4, None, None) == lq.LQ_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 21) + 8)
    assert L.lq_prefill_tokens(h, None, odd, p, p, p, p, 4, None, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_prefill_tokens(h, None, p, p, p, odd, p, 4, None, None) == lq.LQ_ERR_INVALID_ARG   # KDA gate: 16 B
    assert L.lq_prefill_tokens(h, odd, p, p, p, p, p, 4, None, None) == lq.LQ_ERR_INVALID_ARG     # S0: 16 B
    assert L.lq_prefill_tokens(None, None, p, p, p, p, p, 4, None, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_state_destroy(h) == lq.LQ_OK


def test_missing_library_fails_loudly(tmp_path):
    """Without liblq.so the binding raises; there is no fallback path."""
    import subprocess
    import sys
    code = (
        "import sys, torch\n"
        "from recurrent_state_quantization_lq_b200 import lq\n"
        f"lq.LIB_PATH = {str(tmp_path / 'absent' / 'liblq.so')!r}\n"
        "try:\n"
        "    lq.workspace_bytes(lq.make_config(1, 1, 64))\n"
        "except RuntimeError as e:\n"
        "    print('raised', 'missing' in str(e))\n"
        "    sys.exit(0)\n"
        "sys.exit(3)\n"
    )
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "raised True" in r.stdout


def test_resume_validates_on_the_host():
    L = lq.lib()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: resume does no device work
    for kw, ok, bad in (({"window": 8}, (0, 5, 8), (-1, 9)),
                        ({"window": 8, "mode": "naive"}, (0,), (1,)),
                        ({"window": 8, "mode": "fp32"}, (0,), (1,)),
                        ({"window": 8, "ragged": True}, (0,), (1,))):
        cfg = lq.make_config(2, 3, 64, **kw)
        h = ctypes.c_void_p()
        assert L.lq_state_create(ctypes.byref(cfg), fake, lq.workspace_bytes(cfg), ctypes.byref(h)) == lq.LQ_OK
        for n in ok:
            assert L.lq_state_resume(h, n) == lq.LQ_OK, (kw, n)
        for n in bad:
            assert L.lq_state_resume(h, n) == lq.LQ_ERR_INVALID_ARG, (kw, n)
        if not kw.get("ragged") and kw.get("mode", "window") == "window":
            L.lq_state_resume(h, 5)
            assert L.lq_window_fill(h) == 5
        assert L.lq_state_destroy(h) == lq.LQ_OK
    assert L.lq_state_resume(None, 0) == lq.LQ_ERR_INVALID_ARG


def test_export_struct_matches_the_header():
    """The binding's lq_export fields are the header's, in the header's order."""
    import re
    with open(lq.HEADER) as f:
        text = f.read()
    body = re.search(r"typedef struct lq_export \{(.*?)\} lq_export;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"\*\s*(\w+)\s*;", body)
    assert fields == [n for n, _ in lq.Export._fields_]
    assert ctypes.sizeof(lq.Export) == 8 * len(fields)


def test_export_refusals_without_a_gpu():
    """lq_state_export validates on the host before any copy: a bad handle, a
    NULL destination set, a region the mode lacks, a call before the prefill."""
    L = lq.lib()
    assert L.lq_state_export(None, ctypes.byref(lq.Export()), None) == lq.LQ_ERR_INVALID_ARG
    cfg = lq.make_config(2, 3, 64, window=8)
    n = lq.workspace_bytes(cfg)
    h = ctypes.c_void_p()
    assert L.lq_state_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), n, ctypes.byref(h)) == lq.LQ_OK
    try:
        assert L.lq_state_export(h, None, None) == lq.LQ_ERR_INVALID_ARG
        dst = lq.Export()
        dst.state_f32 = 1 << 21                      # windowed handles keep no FP32 state
        assert L.lq_state_export(h, ctypes.byref(dst), None) == lq.LQ_ERR_INVALID_ARG
        assert "state_f32" in lq.last_error()
        dst = lq.Export()
        dst.codes = 1 << 21
        assert L.lq_state_export(h, ctypes.byref(dst), None) == lq.LQ_ERR_STATE   # before any prefill
    finally:
        L.lq_state_destroy(h)


def test_checked_build_exports_every_declared_symbol():
    """The bounds-checked variant (built by __graft_entry__.build() and
    `python -m recurrent_state_quantization_lq_b200.build --bounds-check`)
    exports the same C ABI."""
    import os
    from recurrent_state_quantization_lq_b200 import build as lqbuild
    if not os.path.exists(lqbuild.LIB_CHECKED):
        pytest.skip("liblq_checked.so not built")
    L = ctypes.CDLL(lqbuild.LIB_CHECKED)
    for n in lq.header_symbols():
        assert hasattr(L, n), n
