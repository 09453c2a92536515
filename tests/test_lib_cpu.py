"""The C-ABI library builds for sm_100a, loads, and exports every entry point the
public headers declare (no GPU: no compute calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for hdr in ("dg.h", "dg_ops.h"):
        src = open(os.path.join(ROOT, "include", hdr)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b(dg_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from block_diffusion_moe_denoise_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_headers_declare_the_entry_points():
    names = _declared()
    for n in ("dg_init", "dg_prefill", "dg_denoise_step", "dg_commit_block", "dg_generate", "dg_workspace_size",
              "dg_op_philox_tokens", "dg_op_route_topk", "dg_op_sample", "dg_op_lm_head"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_the_headers():
    from block_diffusion_moe_denoise_b200 import _ffi
    assert sorted(_ffi.exported_symbols()) == _declared()


def test_host_validation_without_gpu(lib):
    """Pure host logic: shape validation and workspace planning need no device."""
    from block_diffusion_moe_denoise_b200 import _ffi, config_struct
    from synth import FULL, TINY
    L = _ffi.load()
    for cfg, req, cap in ((TINY, 1, 1024), (FULL, 1, 4096 + 512), (FULL, 4, 65536 + 256)):
        n = L.dg_workspace_size(ctypes.byref(config_struct(cfg)), req, cap)
        kv = req * cfg.n_layers * 2 * cfg.n_kv_heads * cap * cfg.head_dim * 2
        assert kv < n < kv + 2 * 1024 ** 3
    bad = config_struct(TINY.with_(head_dim=96))
    assert L.dg_workspace_size(ctypes.byref(bad), 1, 1024) == 0
    assert L.dg_workspace_size(ctypes.byref(config_struct(TINY)), 0, 1024) == 0
    assert L.dg_workspace_size(ctypes.byref(config_struct(TINY)), 9, 1024) == 0
    assert L.dg_workspace_size(ctypes.byref(config_struct(TINY.with_(temperature=-0.5))), 1, 1024) == 0
    assert L.dg_workspace_size(ctypes.byref(config_struct(TINY.with_(temperature=0.7))), 1, 1024) > 0
    assert L.dg_workspace_size(ctypes.byref(config_struct(TINY.with_(ffn_selfcond=100))), 1, 1024) == 0
    assert L.dg_workspace_size(ctypes.byref(config_struct(TINY.with_(ffn_selfcond=256, selfcond_topk=9))), 1,
                               1024) == 0
    n0 = L.dg_workspace_size(ctypes.byref(config_struct(TINY)), 1, 1024)
    assert L.dg_workspace_size(ctypes.byref(config_struct(TINY.with_(ffn_selfcond=256))), 1, 1024) > n0
    assert L.dg_strerror(-3) == b"KV capacity or workspace too small"
    # entry points reject bad arguments before touching the device
    assert L.dg_op_route_topk(None, 4, 300, 2, None, None, None) == -1
    assert L.dg_op_philox_tokens(1, 0, 0, 0, 0, 10, 0, None, None) == -1
    assert L.dg_prefill(None, 0, None, 0) == -1
    assert L.dg_op_lm_sample(None, None, 4, 0.7, 1, 0, 1, 0, None, None, None) == -1
    assert L.dg_op_selfcond(None, 0, None, 4, None, None) == -1


def _c_struct_fields(name):
    """(field, C type) in declaration order of `typedef struct name {...} name;` in dg.h."""
    src = open(os.path.join(ROOT, "include", "dg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    body = re.search(r"typedef struct " + name + r" \{(.*?)\} " + name + ";", src, flags=re.S).group(1)
    out = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        m = re.match(r"(const\s+)?(int|float|void|int64_t|const dg_layer_weights)\s*(.*)", decl, flags=re.S)
        base = ("const " if m.group(1) else "") + m.group(2)
        for part in m.group(3).split(","):
            part = part.strip()
            ptr = part.startswith("*")
            out.append((part.lstrip("*").strip(), base + ("*" if ptr else "")))
    return out


def test_ctypes_structs_match_the_header():
    """The binding's ctypes structures declare the header's fields, in order, with
    matching types (an ABI drift check that needs no GPU)."""
    import ctypes as C
    from block_diffusion_moe_denoise_b200 import _ffi
    ctype = {"int": C.c_int, "float": C.c_float, "const void*": C.c_void_p}
    for name, cls in (("dg_config", _ffi.dg_config), ("dg_layer_weights", _ffi.dg_layer_weights)):
        fields = _c_struct_fields(name)
        assert [f for f, _ in fields] == [f for f, _ in cls._fields_], name
        for (f, t), (_, ct) in zip(fields, cls._fields_):
            assert ctype[t] is ct, (name, f, t)
    w = _c_struct_fields("dg_weights")
    assert [f for f, _ in w] == [f for f, _ in _ffi.dg_weights._fields_]


def test_binding_rejects_unusable_tensors_before_any_call():
    """Host memory where the C ABI wants device memory, a wrong element type, a
    non-contiguous view or too few elements raise in Python, before any C call
    could hand a bad address to a kernel."""
    import torch
    import block_diffusion_moe_denoise_b200 as dgm
    from block_diffusion_moe_denoise_b200 import _check, _host
    from synth import TINY

    class NoCalls:                       # a library whose every entry point fails the test
        def __getattr__(self, name):
            def call(*args):
                raise AssertionError(f"{name} was called")
            return call

    h = object.__new__(dgm.DG)          # no device here: only the argument checks run
    h.cfg, h.lib, h.h = TINY, NoCalls(), None
    with pytest.raises(ValueError, match="device"):
        h.prefill(0, torch.zeros(16, dtype=torch.int32))
    with pytest.raises(ValueError, match="device"):
        h.set_canvas(0, torch.zeros(256, dtype=torch.int32), torch.zeros(256, dtype=torch.uint8), 1)
    with pytest.raises(ValueError, match="device"):
        h.op_lm_head(torch.zeros((4, TINY.d_model)))
    import block_diffusion_moe_denoise_b200._ffi as ffi
    real_load = ffi.load
    ffi.load = lambda: NoCalls()
    try:
        with pytest.raises(ValueError, match="device"):
            dgm.philox_tokens(1, 0, 0, 0, 0, 8, 64, torch.zeros(8, dtype=torch.int32), stream=object())
    finally:
        ffi.load = real_load
    # host buffers of dg_generate
    p = torch.zeros(32, dtype=torch.int32)
    assert _host(p, "p", torch.int32, 32).value == p.data_ptr()
    with pytest.raises(ValueError, match="dtype"):
        _host(torch.zeros(32, dtype=torch.int64), "p", torch.int32)
    with pytest.raises(ValueError, match="contiguous"):
        _host(torch.zeros((8, 8), dtype=torch.int32)[:, ::2], "p", torch.int32)
    with pytest.raises(ValueError, match="at least"):
        _host(p, "out", torch.int32, 64)
    with pytest.raises(ValueError, match="shape"):
        _check(torch.zeros((2, 3)), "k", torch.float32, False, shape=(3, 2))


def _host_as_device(monkeypatch):
    """Let the binding's tensor checks accept host tensors as if they were device
    memory, so the remaining checks (dtype, shape, element count) run on a
    machine without a GPU; and make every library entry point fail the test."""
    import block_diffusion_moe_denoise_b200 as dgm
    import block_diffusion_moe_denoise_b200._ffi as ffi
    real = dgm._check

    def check(t, name, dtype, device, numel=None, shape=None):
        return real(t, name, dtype, bool(getattr(t, "is_cuda", False)), numel, shape)

    class NoCalls:
        def __getattr__(self, name):
            def call(*args):
                raise AssertionError(f"{name} was called")
            return call

    monkeypatch.setattr(dgm, "_check", check)
    monkeypatch.setattr(ffi, "load", lambda: NoCalls())
    return dgm


def test_binding_rejects_wrong_weight_shapes_before_init(monkeypatch):
    """A weight of the wrong shape (here one expert row short, or an output
    projection one head narrow) raises in dg_init's binding before any C call: its TMA
    descriptors would otherwise reach past the end of the tensor."""
    import torch
    from synth import TINY, make_weights
    dgm = _host_as_device(monkeypatch)
    w = make_weights(TINY, seed=0)
    for name, bad in (("w_gate", lambda t: t[:, :-1].contiguous()), ("w_o", lambda t: t[:, :-64].contiguous()),
                      ("ws_down", lambda t: t[:-64].contiguous())):
        ww = {"embed": w["embed"], "final_norm": w["final_norm"],
              "layers": [dict(lw) for lw in w["layers"]]}
        ww["layers"][1][name] = bad(ww["layers"][1][name])
        with pytest.raises(ValueError, match=rf"layers\[1\]\.{name}: expected shape"):
            dgm.DG(TINY, ww, max_requests=1, kv_capacity=512, stream=object())
    ww = {"embed": w["embed"][:, :128].contiguous(), "final_norm": w["final_norm"], "layers": w["layers"]}
    with pytest.raises(ValueError, match="embed: expected shape"):
        dgm.DG(TINY, ww, max_requests=1, kv_capacity=512, stream=object())
    shapes = dgm.weight_shapes(TINY)
    for name, t in w["layers"][0].items():
        assert tuple(t.shape) == shapes[name], name


def test_noalloc_binding_rejects_mismatched_embedding(monkeypatch):
    """dg_op_lm_head_noalloc reads embed as [vocab, d_model] rows of x's width:
    a narrower or 1-D embedding, or a 1-D x, raises before any C call."""
    import torch
    dgm = _host_as_device(monkeypatch)
    T, d, V = 8, 256, 1024
    x = torch.zeros((T, d))
    g = torch.ones(d)
    st, am = torch.zeros((T, 4)), torch.zeros(T, dtype=torch.int32)
    with pytest.raises(ValueError, match="embed: expected shape"):
        dgm.lm_head_noalloc(x, g, torch.zeros((V, d - 64), dtype=torch.bfloat16), 1e-6, st, am, stream=object())
    with pytest.raises(ValueError, match="2-D"):
        dgm.lm_head_noalloc(x, g, torch.zeros(V * d, dtype=torch.bfloat16), 1e-6, st, am, stream=object())
    with pytest.raises(ValueError, match="2-D"):
        dgm.lm_head_noalloc(x.view(-1), g, torch.zeros((V, d), dtype=torch.bfloat16), 1e-6, st, am, stream=object())
    with pytest.raises(ValueError, match="final_norm: expected shape"):
        dgm.lm_head_noalloc(x, torch.ones(d + 64), torch.zeros((V, d), dtype=torch.bfloat16), 1e-6, st, am,
                            stream=object())
