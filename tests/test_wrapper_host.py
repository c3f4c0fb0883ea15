"""Host-side argument checks of the Python wrapper (no GPU).

The C ABI takes raw device pointers and trusts the documented layouts, so the
wrapper must refuse a tensor whose shape does not match before any pointer is
handed over.  The objects are built without a handle (no pe_create), so every
case here has to be refused before the wrapper reaches the C library, except
the well-formed host-buffer calls, which reach it and are refused there for the
missing handle."""
from __future__ import annotations

import pytest
import torch

from vlm_vision_patch_b200 import PatchEmbed, PatchMerger

E, C, TP, P = 64, 3, 2, 14
K = C * TP * P * P


def _pe() -> PatchEmbed:
    pe = PatchEmbed.__new__(PatchEmbed)
    pe.E, pe.C, pe.tp, pe.p, pe.has_bias, pe.K = E, C, TP, P, False, K
    pe.h, pe.dev = None, 0
    return pe


def _pm(E_: int = 64, m: int = 2, H: int = 128) -> PatchMerger:
    pm = PatchMerger.__new__(PatchMerger)
    pm.E, pm.m2, pm.H, pm.D = E_, m * m, H, E_ * m * m
    pm.h, pm.dev = None, 0
    return pm


def z(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


@pytest.mark.parametrize("x", [z(4, K + 1), z(4, K - 8), z(K), z(2, 2, K)])
def test_patches_row_width(x):
    with pytest.raises(ValueError, match="x must be"):
        _pe().forward_patches(x)


@pytest.mark.parametrize("out", [z(4, E + 8), z(5, E), z(4 * E)])
def test_patches_out_shape(out):
    with pytest.raises(ValueError, match="out has shape"):
        _pe().forward_patches(z(4, K), out=out)


def test_patches_pos_shape():
    with pytest.raises(ValueError, match="pos has shape"):
        _pe().forward_patches(z(4, K), out=z(4, E), pos=z(4, E - 8))


@pytest.mark.parametrize("frames", [z(3, 28, 28), z(1, 4, 28, 28), z(1, 1, 3, 28, 28)])
def test_frames_layout(frames):
    with pytest.raises(ValueError, match="frames must be"):
        _pe().forward_frames(frames, (1, 2, 2))


def test_frames_grid_and_out():
    with pytest.raises(ValueError, match="grid_thw"):
        _pe().forward_frames(z(1, C, 28, 28), (1, 2))
    with pytest.raises(ValueError, match="out has shape"):
        _pe().forward_frames(z(1, C, 28, 28), (1, 2, 2), out=z(5, E))


def test_grouped_item_lists():
    pe = _pe()
    f = z(1, C, 28, 28)
    with pytest.raises(ValueError, match="one per item"):
        pe.forward_frames_grouped([], [])
    with pytest.raises(ValueError, match="one per item"):
        pe.forward_frames_grouped([f, f], [(1, 2, 2)])
    with pytest.raises(ValueError, match="one per item"):
        pe.forward_frames_grouped([f], [(1, 2, 2), (1, 2, 2)])
    with pytest.raises(ValueError, match=r"\(t, h, w\)"):
        pe.forward_frames_grouped([f], [(1, 2)])
    with pytest.raises(TypeError, match="one dtype"):
        pe.forward_frames_grouped([f, z(1, C, 28, 28, dtype=torch.float32)], [(1, 2, 2), (1, 2, 2)])
    with pytest.raises(ValueError, match="out has shape"):
        pe.forward_frames_grouped([f, f], [(1, 2, 2), (1, 2, 2)], out=z(4, E))
    with pytest.raises(ValueError, match="pos has shape"):
        pe.forward_frames_grouped([f, f], [(1, 2, 2), (1, 2, 2)], out=z(8, E), pos=z(4, E))
    with pytest.raises(ValueError, match="one per item"):
        pe.patchify([f], [])


def test_weight_and_bias_shapes():
    pe = _pe()
    with pytest.raises(ValueError, match="weight has shape"):
        pe.set_weight(z(E, C, TP, P, P - 1))
    with pytest.raises(ValueError, match="weight has shape"):
        pe.set_weight(z(E + 8, K))
    with pytest.raises(ValueError, match="bias has shape"):
        pe.set_weight(z(E, C, TP, P, P), z(E + 1))


def test_cpu_tensors_are_refused_after_the_shape_checks():
    """Shapes right, memory wrong: the pointer check still stops the call."""
    with pytest.raises(ValueError, match="CUDA tensor"):
        _pe().forward_patches(z(4, K), out=z(4, E))


def test_merger_shapes():
    pm = _pm()
    with pytest.raises(ValueError, match="x must be"):
        pm.forward(z(8, 72))
    with pytest.raises(ValueError, match="out has shape"):
        pm.forward(z(8, 64), out=z(3, 128))
    good = dict(gamma=z(64), beta=z(64), w1=z(256, 256), b1=None, w2=z(128, 256), b2=None)
    for name, bad in (("gamma", z(63)), ("beta", z(64, 1)), ("w1", z(256, 255)), ("b1", z(255)),
                      ("w2", z(256, 128)), ("b2", z(127))):
        kw = dict(good, **{name: bad})
        with pytest.raises(ValueError, match=f"{name} has shape"):
            pm.set_weights(**kw)


def test_host_buffer_calls_check_shapes_then_reach_the_library():
    from vlm_vision_patch_b200 import PEError
    pe = _pe()
    with pytest.raises(ValueError, match="x must be"):
        pe.forward_patches_host(z(4, K + 2))
    with pytest.raises(ValueError, match="out has shape"):
        pe.forward_patches_host(z(4, K), out=z(4, E + 8))
    f = z(1, C, 28, 28)
    with pytest.raises(ValueError, match="one per item"):
        pe.forward_frames_grouped_host([f], [(1, 2, 2), (1, 2, 2)])
    with pytest.raises(ValueError, match="out has shape"):
        pe.forward_frames_grouped_host([f], [(1, 2, 2)], out=z(3, E))
    # well-formed host tensors reach the C call (raw stream handle 0: no CUDA
    # query on the way), which refuses the missing handle
    with pytest.raises(PEError) as e:
        pe.forward_patches_host(z(4, K), stream=0, blocking=False)
    assert e.value.status == "PE_ERR_INVALID_ARG"
    with pytest.raises(PEError) as e:
        pe.forward_frames_grouped_host([f], [(1, 2, 2)], stream=0, blocking=False)
    assert e.value.status == "PE_ERR_INVALID_ARG"
