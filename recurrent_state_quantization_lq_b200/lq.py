"""Thin Python binding of liblq (include/lq.h): argument marshalling only.

Every step of the decode path runs in liblq's CUDA kernels; PyTorch supplies
device memory (the workspace and the input/output tensors) and streams.  If
liblq.so has not been built, importing the library raises: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LQ_LIBRARY may name another build of the same C ABI, e.g. the bounds-checked
# liblq_checked.so (python -m recurrent_state_quantization_lq_b200.build --bounds-check)
LIB_PATH = os.environ.get("LQ_LIBRARY") or os.path.join(_HERE, "liblq.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "lq.h")

# enums of include/lq.h
LQ_OK, LQ_ERR_INVALID_ARG, LQ_ERR_UNSUPPORTED, LQ_ERR_WORKSPACE, LQ_ERR_WINDOW_FULL = 0, 1, 2, 3, 4
LQ_ERR_RANGE, LQ_ERR_CUDA, LQ_ERR_DEVICE, LQ_ERR_STATE = 5, 6, 7, 8
GATE = {"scalar": 0, "gdn": 0, "channel": 1, "kda": 1}
MODE = {"window": 0, "naive": 1, "fp32": 2}
SELECT = {"l2": 0, "maxabs": 1}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
ABSENT = ctypes.c_size_t(-1).value

LQ_DEVERR_BOUNDS = 4   # device error code: an index out of range (checked build; unit tickets in every build)

STATUS_NAMES = {0: "LQ_OK", 1: "LQ_ERR_INVALID_ARG", 2: "LQ_ERR_UNSUPPORTED", 3: "LQ_ERR_WORKSPACE",
                4: "LQ_ERR_WINDOW_FULL", 5: "LQ_ERR_RANGE", 6: "LQ_ERR_CUDA", 7: "LQ_ERR_DEVICE",
                8: "LQ_ERR_STATE"}


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "heads", "d_k", "d_v", "window", "n_comp_rows", "n_comp_cols", "gate", "mode",
        "smooth", "select", "in_dtype", "ragged")]


class Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "total_bytes", "err", "codes", "row_scale", "col_smooth", "comp_index", "comp_row_vec",
        "comp_col_vec", "gate_sum", "buf_delta", "buf_key", "buf_gate", "state_f32")] + \
        [("comp_index_stride", ctypes.c_int32), ("window_pad", ctypes.c_int32), ("fill", ctypes.c_size_t)]


EXPORT_REGIONS = ("codes", "row_scale", "col_smooth", "comp_index", "comp_row_vec", "comp_col_vec", "buf_delta",
                  "buf_key", "buf_gate", "gate_sum", "fill", "state_f32")


class Export(ctypes.Structure):
    """lq_export: destination pointers of lq_state_export (NULL = not copied)."""
    _fields_ = [(n, ctypes.c_void_p) for n in EXPORT_REGIONS]


class LQError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}: {last_error()}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load liblq.so (built in-tree by ``python -m recurrent_state_quantization_lq_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m recurrent_state_quantization_lq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32 = ctypes.c_void_p, ctypes.c_int32
        L.lq_workspace_bytes.argtypes = [ctypes.POINTER(Config)]
        L.lq_workspace_bytes.restype = ctypes.c_size_t
        L.lq_workspace_layout.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Layout)]
        L.lq_workspace_layout.restype = i32
        L.lq_state_create.argtypes = [ctypes.POINTER(Config), vp, ctypes.c_size_t, ctypes.POINTER(vp)]
        L.lq_state_create.restype = i32
        L.lq_prefill_state.argtypes = [vp, vp, vp]
        L.lq_prefill_state.restype = i32
        L.lq_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
        L.lq_decode_step.restype = i32
        L.lq_decode_step_active.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.lq_decode_step_active.restype = i32
        L.lq_window_flush.argtypes = [vp, vp]
        L.lq_window_flush.restype = i32
        L.lq_window_flush_pending.argtypes = [vp, vp]
        L.lq_window_flush_pending.restype = i32
        L.lq_prefill_sequences.argtypes = [vp, vp, vp, vp]
        L.lq_prefill_sequences.restype = i32
        L.lq_prefill_tokens.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, vp]
        L.lq_prefill_tokens.restype = i32
        L.lq_prefill_sequences_tokens.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp]
        L.lq_prefill_sequences_tokens.restype = i32
        L.lq_state_resume.argtypes = [vp, i32]
        L.lq_state_resume.restype = i32
        L.lq_window_fill.argtypes = [vp]
        L.lq_window_fill.restype = i32
        L.lq_state_export.argtypes = [vp, ctypes.POINTER(Export), vp]
        L.lq_state_export.restype = i32
        L.lq_device_status.argtypes = [vp, vp]
        L.lq_device_status.restype = i32
        L.lq_state_destroy.argtypes = [vp]
        L.lq_state_destroy.restype = i32
        L.lq_last_error_string.argtypes = []
        L.lq_last_error_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Names of the entry points include/lq.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"LQ_API\s+[\w\s\*]+?\b(lq_\w+)\s*\(", text)


def last_error() -> str:
    return lib().lq_last_error_string().decode()


def make_config(batch: int, heads: int, d: int, window: int = 64, n_comp_rows: int = 2,
                n_comp_cols: int = 2, gate: str = "scalar", mode: str = "window", smooth: int = 1,
                select: str = "l2", in_dtype: torch.dtype = torch.bfloat16, ragged: bool = False) -> Config:
    return Config(batch, heads, d, d, window, n_comp_rows, n_comp_cols, GATE[gate], MODE[mode],
                  smooth, SELECT[select], DTYPE[in_dtype], int(ragged))


def workspace_bytes(cfg: Config) -> int:
    return lib().lq_workspace_bytes(ctypes.byref(cfg))


def workspace_layout(cfg: Config) -> Layout:
    L = Layout()
    st = lib().lq_workspace_layout(ctypes.byref(cfg), ctypes.byref(L))
    if st != LQ_OK:
        raise LQError(st, "lq_workspace_layout")
    return L


def _stream_ptr(stream, device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(None if t is None else t.data_ptr())


class DecodeState:
    """A batch of (sequence, head) recurrent states of one layer, held by liblq.

    The workspace is a torch uint8 tensor on ``device``; its regions can be
    viewed with :meth:`view`.  All calls enqueue on ``stream`` (default: the
    current stream) and return without synchronizing.
    """

    def __init__(self, batch: int, heads: int, d: int, *, window: int = 64, n_comp_rows: int = 2,
                 n_comp_cols: int = 2, gate: str = "scalar", mode: str = "window", smooth: int = 1,
                 select: str = "l2", in_dtype: torch.dtype = torch.bfloat16, ragged: bool = False,
                 device=None):
        self.cfg = make_config(batch, heads, d, window, n_comp_rows, n_comp_cols, gate, mode, smooth,
                               select, in_dtype, ragged)
        self.ragged = bool(ragged)
        dev = torch.device(device) if device is not None else torch.device("cuda")
        if dev.index is None:
            dev = torch.device(dev.type, torch.cuda.current_device())
        self.device = dev
        nbytes = workspace_bytes(self.cfg)
        if nbytes == 0:
            raise LQError(LQ_ERR_INVALID_ARG, "lq_workspace_bytes")
        self.layout = workspace_layout(self.cfg)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        st = lib().lq_state_create(ctypes.byref(self.cfg), _ptr(self.workspace), nbytes, ctypes.byref(h))
        if st != LQ_OK:
            raise LQError(st, "lq_state_create")
        self._h = h
        self.batch, self.heads, self.d = batch, heads, d
        self.in_dtype = in_dtype
        self.per_channel_gate = GATE[gate] == 1

    # ------------------------------------------------------------------ calls
    def _check(self, st: int, what: str) -> None:
        if st != LQ_OK:
            raise LQError(st, what)

    def prefill(self, S0: torch.Tensor | None = None, stream=None) -> None:
        if S0 is not None:
            assert S0.dtype == torch.float32 and S0.is_contiguous() and S0.device == self.device
            assert S0.numel() == self.batch * self.heads * self.d * self.d
        self._check(lib().lq_prefill_state(self._h, _ptr(S0), _stream_ptr(stream, self.device)),
                    "lq_prefill_state")

    def decode_step(self, q, k, v, g, beta, out: torch.Tensor | None = None, stream=None,
                    active: torch.Tensor | None = None) -> torch.Tensor:
        """One token for every sequence; on a ragged state, for the sequences
        with active[b] != 0 (uint8 [batch] on the device; None = all)."""
        if out is None:
            out = torch.empty(self.batch, self.heads, self.d, dtype=torch.float32, device=self.device)
        for t, dt in ((q, self.in_dtype), (k, self.in_dtype), (v, self.in_dtype), (g, torch.float32),
                      (beta, torch.float32), (out, torch.float32)):
            assert t.dtype == dt and t.is_contiguous() and t.device == self.device, (t.dtype, t.device)
        if active is not None:
            assert active.dtype == torch.uint8 and active.numel() == self.batch and active.device == self.device
            self._check(lib().lq_decode_step_active(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                                    _ptr(active), _ptr(out), _stream_ptr(stream, self.device)),
                        "lq_decode_step_active")
        else:
            self._check(lib().lq_decode_step(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(out),
                                             _stream_ptr(stream, self.device)), "lq_decode_step")
        return out

    def flush(self, stream=None) -> None:
        """End the window (ragged: of every unit whose window is full)."""
        self._check(lib().lq_window_flush(self._h, _stream_ptr(stream, self.device)), "lq_window_flush")

    def flush_pending(self, stream=None) -> None:
        """Ragged: end the window of every unit holding buffered tokens."""
        self._check(lib().lq_window_flush_pending(self._h, _stream_ptr(stream, self.device)),
                    "lq_window_flush_pending")

    def prefill_sequences(self, S0: torch.Tensor | None, mask: torch.Tensor, stream=None) -> None:
        """Ragged: restart the sequences with mask[b] != 0 (uint8 [batch] on the
        device) from S0 (FP32 [batch, heads, d, d]; None = zero state)."""
        if S0 is not None:
            assert S0.dtype == torch.float32 and S0.is_contiguous() and S0.device == self.device
            assert S0.numel() == self.batch * self.heads * self.d * self.d
        assert mask.dtype == torch.uint8 and mask.numel() == self.batch and mask.device == self.device
        self._check(lib().lq_prefill_sequences(self._h, _ptr(S0), _ptr(mask), _stream_ptr(stream, self.device)),
                    "lq_prefill_sequences")

    def prefill_tokens(self, q, k, v, g, beta, S0: torch.Tensor | None = None, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor | None:
        """Run the FP32 recurrence over a prompt (inputs [T, batch, heads, ...]
        as for decode_step, stacked over tokens) from S0 (None = zero state) and
        encode its final state as the window-start state.  Writes the prompt's
        outputs into `out` ([T, batch, heads, d] FP32) when given."""
        T = q.shape[0]
        for t, dt in ((q, self.in_dtype), (k, self.in_dtype), (v, self.in_dtype), (g, torch.float32),
                      (beta, torch.float32)):
            assert t.dtype == dt and t.is_contiguous() and t.device == self.device and t.shape[0] == T, t.dtype
        if out is not None:
            assert out.dtype == torch.float32 and out.is_contiguous() and out.device == self.device
            assert out.numel() == T * self.batch * self.heads * self.d
        if S0 is not None:
            assert S0.dtype == torch.float32 and S0.is_contiguous() and S0.device == self.device
            assert S0.numel() == self.batch * self.heads * self.d * self.d
        self._check(lib().lq_prefill_tokens(self._h, _ptr(S0), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), T,
                                            _ptr(out), _stream_ptr(stream, self.device)), "lq_prefill_tokens")
        return out

    def prefill_sequences_tokens(self, q, k, v, g, beta, mask: torch.Tensor, lengths: torch.Tensor | None = None,
                                 S0: torch.Tensor | None = None, out: torch.Tensor | None = None,
                                 stream=None) -> torch.Tensor | None:
        """Ragged: restart the sequences with mask[b] != 0 from S0 (None = zero)
        through their prompts: inputs [T, batch, heads, ...] padded to T tokens,
        lengths int32 [batch] on the device (None = T for every sequence)."""
        T = q.shape[0]
        for t, dt in ((q, self.in_dtype), (k, self.in_dtype), (v, self.in_dtype), (g, torch.float32),
                      (beta, torch.float32)):
            assert t.dtype == dt and t.is_contiguous() and t.device == self.device and t.shape[0] == T, t.dtype
        assert mask.dtype == torch.uint8 and mask.numel() == self.batch and mask.device == self.device
        if lengths is not None:
            assert lengths.dtype == torch.int32 and lengths.numel() == self.batch and lengths.device == self.device
        if out is not None:
            assert out.dtype == torch.float32 and out.is_contiguous() and out.device == self.device
            assert out.numel() == T * self.batch * self.heads * self.d
        if S0 is not None:
            assert S0.dtype == torch.float32 and S0.is_contiguous() and S0.device == self.device
            assert S0.numel() == self.batch * self.heads * self.d * self.d
        self._check(lib().lq_prefill_sequences_tokens(self._h, _ptr(S0), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                                      _ptr(beta), T, _ptr(lengths), _ptr(mask), _ptr(out),
                                                      _stream_ptr(stream, self.device)),
                    "lq_prefill_sequences_tokens")
        return out

    def checkpoint(self, stream=None) -> tuple[torch.Tensor, int]:
        """A copy of the whole state: the workspace bytes and the shared-window
        count (0 on a ragged state, whose counts are in the workspace)."""
        status = self.device_status(stream)
        if status != LQ_OK:
            raise LQError(status, "checkpoint of a state with a device error")
        return self.workspace.clone(), max(self.fill, 0)

    def resume(self, workspace: torch.Tensor, n_buf: int) -> None:
        """Continue from a checkpoint() of a state with the same configuration."""
        assert workspace.dtype == torch.uint8 and workspace.numel() == self.workspace.numel()
        self.workspace.copy_(workspace)
        torch.cuda.synchronize(self.device)
        self._check(lib().lq_state_resume(self._h, int(n_buf)), "lq_state_resume")

    @property
    def fill(self) -> int:
        """Tokens buffered in the shared window; -1 on a ragged state (see fills())."""
        return lib().lq_window_fill(self._h)

    def fills(self) -> torch.Tensor:
        """Tokens buffered per (sequence, head) (read through lq_state_export,
        whatever the device error word holds)."""
        return self.export(["fill"], check=False)["fill"]

    def export_shapes(self) -> dict:
        """Dtype and packed shape of every region lq_state_export can copy for
        this state (regions the mode does not keep are absent)."""
        L, c = self.layout, self.cfg
        B, H, d, W = c.batch, c.heads, c.d_k, c.window
        key_dt = torch.float32 if (c.gate == 1 or c.in_dtype == 0) else torch.bfloat16
        spec = {
            "codes": (torch.int8, (B, H, d, d)),
            "row_scale": (torch.float32, (B, H, d)),
            "col_smooth": (torch.float32, (B, H, d)),
            "comp_index": (torch.int32, (B, H, c.n_comp_rows + c.n_comp_cols)),
            "comp_row_vec": (torch.float32, (B, H, c.n_comp_rows, d)),
            "comp_col_vec": (torch.float32, (B, H, c.n_comp_cols, d)),
            "buf_delta": (torch.float32, (B, H, W, d)),
            "buf_key": (key_dt, (B, H, W, d)),
            "buf_gate": (torch.float32, (B, H, W)),
            "gate_sum": (torch.float64, (B, H, d if c.gate == 1 else 1)),
            "fill": (torch.int32, (B, H)),
            "state_f32": (torch.float32, (B, H, d, d)),
        }
        present = {n for n in EXPORT_REGIONS if n != "fill" and getattr(L, n) != ABSENT}
        if c.mode == MODE["window"]:
            present.add("fill")
        return {n: spec[n] for n in EXPORT_REGIONS if n in present}

    def export(self, names=None, device="cpu", stream=None, check: bool = True) -> dict:
        """Copy state regions out through lq_state_export into new tensors on
        `device` (host tensors are pinned).  names: regions to copy (None = all
        this state keeps).  Synchronizes the stream.  Raises LQError when the
        device error word is set, unless check is False."""
        shapes = self.export_shapes()
        names = list(shapes) if names is None else list(names)
        dev = torch.device(device)
        pin = dev.type == "cpu" and torch.cuda.is_available()
        out, dst = {}, Export()
        for n in names:
            if n not in shapes:
                raise KeyError(f"this state keeps no {n}")
            dt, shape = shapes[n]
            x = torch.empty(shape, dtype=dt, device=dev, pin_memory=pin)
            out[n] = x
            if x.numel():
                setattr(dst, n, x.data_ptr())
        st = lib().lq_state_export(self._h, ctypes.byref(dst), _stream_ptr(stream, self.device))
        if st != LQ_OK and (check or st in (LQ_ERR_INVALID_ARG, LQ_ERR_STATE, LQ_ERR_CUDA)):
            raise LQError(st, "lq_state_export")
        return out

    def read(self, name: str, device="cpu", check: bool = True) -> torch.Tensor:
        """One region of the state, copied out through lq_state_export."""
        return self.export([name], device=device, check=check)[name]

    def device_status(self, stream=None) -> int:
        """Synchronize and return the status of the device error word (LQ_OK if clean)."""
        return lib().lq_device_status(self._h, _stream_ptr(stream, self.device))

    # ------------------------------------------------------------ inspection
    def view(self, name: str) -> torch.Tensor | None:
        """A writable tensor view of one workspace region, laid out as lq_layout
        says (internal layout: read the state with export(); this is for
        writing a state in, as a checkpoint restore does)."""
        L, c = self.layout, self.cfg
        off = getattr(L, name)
        if off == ABSENT:
            return None
        N, d = c.batch * c.heads, c.d_k
        gd = d if c.gate == 1 else 1
        key_dt = torch.float32 if (c.gate == 1 or c.in_dtype == 0) else torch.bfloat16
        nc = L.comp_index_stride
        spec = {
            "err": (torch.int32, (64,)),
            "codes": (torch.int8, (c.batch, c.heads, d, d)),
            "row_scale": (torch.float32, (c.batch, c.heads, d)),
            "col_smooth": (torch.float32, (c.batch, c.heads, d)),
            "comp_index": (torch.int32, (c.batch, c.heads, nc)),
            "comp_row_vec": (torch.float32, (c.batch, c.heads, c.n_comp_rows, d)),
            "comp_col_vec": (torch.float32, (c.batch, c.heads, c.n_comp_cols, d)),
            "gate_sum": (torch.float64, (c.batch, c.heads, gd)),
            "buf_delta": (torch.float32, (c.batch, c.heads, c.window, d)),
            "buf_key": (key_dt, (c.batch, c.heads, c.window, d)),
            "buf_gate": (torch.float32, (c.batch, c.heads, L.window_pad)),
            "state_f32": (torch.float32, (c.batch, c.heads, d, d)),
            "fill": (torch.int32, (c.batch, c.heads)),
        }[name]
        dt, shape = spec
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dt).element_size()
        return self.workspace[off:off + nbytes].view(dt).view(shape)

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().lq_state_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
