"""Host-side checks of the C ABI (no GPU needed): the library builds, loads,
and exports every function include/m3.h declares; argument validation that
happens before any CUDA call returns status codes."""
import ctypes as C
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header=None):
    """The functions include/*.h declare (or one header's)."""
    inc = os.path.join(ROOT, "include")
    names = set()
    for h in sorted(os.listdir(inc)):
        if header is None or h == header:
            src = open(os.path.join(inc, h)).read()
            names |= set(re.findall(r"^M3_API\s+[\w\s\*]+?\b(m3_\w+)\s*\(", src, re.M))
    return sorted(names)


def test_header_declares_the_abi():
    names = _declared()
    for n in ("m3_create", "m3_load_weights", "m3_kv_alloc", "m3_decode_frame", "m3_depth_decode"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from autoregressive_audio_token_b200 import build
    path = build.build()
    lib = C.CDLL(path)
    for n in _declared():
        assert hasattr(lib, n), n


def test_binding_covers_the_abi():
    from autoregressive_audio_token_b200 import dit, m3
    assert sorted(m3.EXPORTED) == _declared("m3.h")
    assert sorted(dit.EXPORTED) == _declared("m3_dit.h")
    for n in _declared("m3.h"):
        assert hasattr(m3, n), n
    for n in _declared("m3_dit.h"):
        assert hasattr(dit, n), n


def test_dit_create_rejects_unsupported_shapes_without_gpu():
    import synth
    from autoregressive_audio_token_b200 import dit, m3
    for bad in ({"head_dim": 128}, {"rope_dims": 16}, {"width": 384, "n_heads": 6},
                {"ffn": 100}, {"temb": 12}, {"latent": 12}):
        import dataclasses
        s = dataclasses.replace(synth.DIT, **bad)
        d = C.c_void_p()
        rc = m3.lib.m3_dit_create(C.byref(dit.config_from_shape(s, 689)), None, C.byref(d))
        assert rc == m3.M3_EINVAL, bad
        assert b"m3_dit_config" in m3.lib.m3_last_error()
    assert m3.lib.m3_dit_step(None, 1, None, None, None, 1.0, 0.9, 1.7, None, None) == m3.M3_EINVAL


def test_create_rejects_bad_config_without_gpu():
    from autoregressive_audio_token_b200 import m3
    cfg = m3.m3_config()
    cfg.hidden = 100  # not a multiple of 16, head_dim 0
    ctx = C.c_void_p()
    rc = m3.lib.m3_create(C.byref(cfg), None, C.byref(ctx))
    assert rc == m3.M3_EINVAL
    assert b"m3_config" in m3.lib.m3_last_error()


def test_null_arguments_are_einval():
    from autoregressive_audio_token_b200 import m3
    assert m3.lib.m3_decode_frame(None, 1, None, 0, 0, None, 0.0, 1.0, None, None, None) == m3.M3_EINVAL
    assert m3.lib.m3_quantize_int8(None, 1, 1, 1, None, None, None) == m3.M3_EINVAL
    assert m3.lib.m3_depth_decode(None, 2, None, None, 0, 0, 1.5, 1.0, None, None, None) == m3.M3_EINVAL
    # launch accounting answers without a context only with an error
    assert m3.lib.m3_frame_kernels(None, 1) == m3.M3_EINVAL
    assert m3.lib.m3_depth_kernels(None, 1) == m3.M3_EINVAL


def test_checking_hooks_validate_before_any_cuda_call():
    from autoregressive_audio_token_b200 import m3
    assert m3.lib.m3_inject_fault(None, m3.M3_FAULT_ALLOC, 1) == m3.M3_EINVAL
    assert m3.lib.m3_stalled_wait(None, 10) == m3.M3_EINVAL
    assert m3.lib.m3_gumbel_fill(1, 2, 3, 4, -1, None, None) == m3.M3_EINVAL
    assert m3.lib.m3_gumbel_fill(1, 2, 3, 4, 5, None, None) == m3.M3_EINVAL
    assert m3.lib.m3_gumbel_fill(1, 2, 3, 4, 0, None, None) == m3.M3_OK  # nothing to do
