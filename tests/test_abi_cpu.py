"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import gen
import sparse_moe_layer_renormalised_b200 as moe
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    src = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)


def _dims(**kw):
    base = dict(T=128, H=2048, L=1024, E=128, k=8, I=768, S=2, Is=1024)
    base.update(kw)
    return moe.Dims(**base)


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) == 23
    lib = ctypes.CDLL(moe.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(moe.EXPORTED)


def test_status_strings():
    assert moe.moe_status_str(0) == "MOE_OK"
    assert moe.moe_status_str(2) == "MOE_ERR_UNSUPPORTED"


def test_workspace_size():
    assert moe.moe_workspace_size(_dims(k=200)) == 0
    a = moe.moe_workspace_size(_dims(T=100))
    b = moe.moe_workspace_size(_dims(T=1000))
    assert 0 < a < b
    k3 = moe.moe_workspace_size(_dims(T=16384, H=7168, L=3584, E=896, k=16, I=3072, S=2, Is=3072))
    # dominated by the permuted latent rows (bf16), expert h (bf16) and y_perm (fp32)
    R = 16384 * 16
    assert k3 >= R * (3584 * 2 + 3072 * 2 + 3584 * 4)


FAKE = 1 << 20  # an aligned address; never dereferenced because validation fails first


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(k=129, E=128), moe.MOE_ERR_INVALID_ARG),
    (dict(k=33, E=128), moe.MOE_ERR_INVALID_ARG),
    (dict(E=1025), moe.MOE_ERR_INVALID_ARG),
    (dict(T=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(L=1020), moe.MOE_ERR_INVALID_ARG),
    (dict(situ_c=0.0), moe.MOE_ERR_INVALID_ARG),
    (dict(y_out="mxfp4"), moe.MOE_ERR_INVALID_ARG),
    (dict(routed="mxfp4"), moe.MOE_ERR_UNSUPPORTED),  # L = 1024 fine, I = 768 not a multiple of 512
    (dict(routed="mxfp4", act="f32", y_out="f32"), moe.MOE_ERR_UNSUPPORTED),
    (dict(routed="mxfp4_a8"), moe.MOE_ERR_UNSUPPORTED),  # I = 768 not a multiple of 512
    (dict(routed="mxfp4_a8", I=1024, act="f32", y_out="f32"), moe.MOE_ERR_UNSUPPORTED),
    (dict(routed="mxfp4_a4"), moe.MOE_ERR_UNSUPPORTED),  # I = 768 not a multiple of 512
    (dict(routed="mxfp4_a4", I=1024, act="f32", y_out="f32"), moe.MOE_ERR_UNSUPPORTED),
    (dict(H=2056), moe.MOE_ERR_UNSUPPORTED),
    (dict(S=4), moe.MOE_ERR_UNSUPPORTED),
])
def test_invalid_dims_rejected(kw, status):
    d = _dims(**kw)
    w = moe.make_weights(**{f: FAKE for f in ("Wr", "bias", "Wdown", "Wup", "gamma", "Wg", "Wv", "Wo", "Wsg", "Wsv",
                                                "Wso")})
    assert moe.moe_layer_forward(d, w, FAKE, FAKE, None, FAKE, 1 << 40, 0) == status


def test_bad_pointers_rejected():
    d = _dims()
    full = {f: FAKE for f in ("Wr", "bias", "Wdown", "Wup", "gamma", "Wg", "Wv", "Wo", "Wsg", "Wsv", "Wso")}
    ws = moe.moe_workspace_size(d)
    for f in full:
        w = moe.make_weights(**{**full, f: None})
        assert moe.moe_layer_forward(d, w, FAKE, FAKE, None, FAKE, ws, 0) == moe.MOE_ERR_INVALID_ARG, f
        w = moe.make_weights(**{**full, f: FAKE + 8})
        assert moe.moe_layer_forward(d, w, FAKE, FAKE, None, FAKE, ws, 0) == moe.MOE_ERR_INVALID_ARG, f
    w = moe.make_weights(**full)
    assert moe.moe_layer_forward(d, w, None, FAKE, None, FAKE, ws, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_layer_forward(d, w, FAKE, FAKE, None, FAKE + 16, ws, 0) == moe.MOE_ERR_INVALID_ARG  # ws alignment
    assert moe.moe_layer_forward(d, w, FAKE, FAKE, None, FAKE, ws - 1, 0) == moe.MOE_ERR_INVALID_ARG  # ws size
    aux = moe.make_aux(u=FAKE + 4)
    assert moe.moe_layer_forward(d, w, FAKE, FAKE, aux, FAKE, ws, 0) == moe.MOE_ERR_INVALID_ARG
    w_scaled = moe.make_weights(**{**full, "Sg": FAKE})  # scales with bf16 weights
    assert moe.moe_layer_forward(d, w_scaled, FAKE, FAKE, None, FAKE, ws, 0) == moe.MOE_ERR_INVALID_ARG
    dm = _dims(I=1024, routed="mxfp4")
    wsm = moe.moe_workspace_size(dm)
    assert moe.moe_layer_forward(dm, w, FAKE, FAKE, None, FAKE, wsm, 0) == moe.MOE_ERR_INVALID_ARG  # no scales
    wm = moe.make_weights(**{**full, "Sg": FAKE, "Sv": FAKE, "So": FAKE + 4})
    assert moe.moe_layer_forward(dm, wm, FAKE, FAKE, None, FAKE, wsm, 0) == moe.MOE_ERR_INVALID_ARG  # misaligned


def test_stage_entry_points_validate():
    d = _dims()
    ws = moe.moe_workspace_size(d)
    assert moe.moe_router_topk(d, None, None, FAKE, FAKE, 0, FAKE, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_router_topk(d, None, None, None, FAKE, 1, FAKE, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_permute(d, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_permute(d, FAKE, None, FAKE, FAKE, FAKE, None, FAKE, 10, 0) == moe.MOE_ERR_INVALID_ARG
    w = moe.make_weights(Wg=FAKE, Wv=FAKE)
    assert moe.moe_expert_ffn(d, w, FAKE, FAKE, FAKE, FAKE, ws, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_combine(d, FAKE, FAKE, FAKE, None, None, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_combine(d, FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, 0) == moe.MOE_ERR_INVALID_ARG


def test_qb_bias_update_validates():
    """Bad dims, bins, range and pointers are rejected on the host (the
    pointers are never dereferenced)."""
    ok = dict(scores=FAKE, bias_in=FAKE, bias_out=FAKE, quantile_out=None, hist=FAKE, nbins=256, lo=-1.0, hi=1.0)

    def call(d=None, **kw):
        a = {**ok, **kw}
        return moe.moe_qb_bias_update(d or _dims(), a["scores"], a["bias_in"], a["bias_out"], a["quantile_out"],
                                      a["hist"], a["nbins"], a["lo"], a["hi"], 0)

    assert call(d=_dims(E=1, k=1)) == moe.MOE_ERR_INVALID_ARG       # k must be < E
    assert call(d=_dims(E=2048)) == moe.MOE_ERR_INVALID_ARG         # E > 1024
    assert call(d=_dims(T=4, E=128, k=8)) == moe.MOE_ERR_INVALID_ARG  # target floor(T k / E) = 0
    assert call(nbins=100) == moe.MOE_ERR_INVALID_ARG                # not a multiple of 32
    assert call(nbins=1 << 17) == moe.MOE_ERR_INVALID_ARG
    assert call(lo=1.0, hi=1.0) == moe.MOE_ERR_INVALID_ARG
    assert call(hi=float("inf")) == moe.MOE_ERR_INVALID_ARG
    assert call(hist=None) == moe.MOE_ERR_INVALID_ARG
    assert call(scores=FAKE + 2) == moe.MOE_ERR_INVALID_ARG           # misaligned


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import sparse_moe_layer_renormalised_b200._binding as b

    monkeypatch.setattr(b, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(b, "_lib", None)
    with pytest.raises(moe.MoeLibraryMissing):
        b.lib()


def test_stage_entry_points_validate_before_launching():
    """moe_latent_shared / moe_output / moe_expert_ffn_blocks reject bad
    arguments on the host (no GPU needed: nothing is launched)."""
    d = _dims(T=64)
    w = moe.make_weights(Wdown=FAKE, Wup=FAKE, Wsg=FAKE, Wsv=FAKE, Wso=FAKE, Wg=FAKE, Wv=FAKE, Wo=FAKE)
    assert moe.moe_latent_shared(d, w, None, FAKE, FAKE) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_latent_shared(d, w, FAKE + 4, FAKE, FAKE) == moe.MOE_ERR_INVALID_ARG  # misaligned x
    assert moe.moe_output(d, w, FAKE, None, FAKE) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_output(_dims(k=200), w, FAKE, FAKE, FAKE) == moe.MOE_ERR_INVALID_ARG
    n = moe.moe_expert_ffn_blocks_workspace_size(d, 1000, 4)
    assert n > 0 and n > moe.moe_expert_ffn_blocks_workspace_size(d, 1000, 1)
    assert moe.moe_expert_ffn_blocks_workspace_size(d, 1000, 0) == 0
    assert moe.moe_expert_ffn_blocks(d, w, FAKE, 1000, FAKE, 0, FAKE, FAKE, n) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_expert_ffn_blocks(d, w, FAKE, 1000, FAKE, 4, FAKE, FAKE, n - 1) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_expert_ffn_blocks(d, w, FAKE, -1, FAKE, 4, FAKE, FAKE, n) == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("routed", ["mxfp4_a8", "mxfp4_a4"])
def test_block_scaled_path_validates(routed):
    """The block-scaled routed types need the tiled weight scales and 32-byte
    aligned codes; tiled scales on any other path are rejected; the size query
    and the tiling and quantiser entries validate on the host."""
    full = {f: FAKE for f in ("Wr", "bias", "Wdown", "Wup", "gamma", "Wg", "Wv", "Wo", "Wsg", "Wsv", "Wso")}
    d8 = _dims(I=1024, routed=routed)
    ws8 = moe.moe_workspace_size(d8)
    assert ws8 > moe.moe_workspace_size(_dims(I=1024, routed="mxfp4"))  # + the codes of h and the scale tiles
    if routed == "mxfp4_a4":  # h's codes take half the bytes of the MXFP8 path's
        assert ws8 < moe.moe_workspace_size(_dims(I=1024, routed="mxfp4_a8"))
    tiled = dict(Sgv_tiled=FAKE, So_tiled=FAKE)
    call = lambda w: moe.moe_layer_forward(d8, moe.make_weights(**w), FAKE, FAKE, None, FAKE, ws8, 0)  # noqa: E731
    assert call(full) == moe.MOE_ERR_INVALID_ARG                                  # no tiled scales
    assert call({**full, **tiled, "So_tiled": FAKE + 8}) == moe.MOE_ERR_INVALID_ARG  # misaligned
    assert call({**full, **tiled, "Wv": FAKE + 16}) == moe.MOE_ERR_INVALID_ARG       # codes not 32-byte aligned
    dm = _dims(I=1024, routed="mxfp4")
    wsm = moe.moe_workspace_size(dm)
    wm = moe.make_weights(**{**full, "Sg": FAKE, "Sv": FAKE, "So": FAKE, **tiled})
    assert moe.moe_layer_forward(dm, wm, FAKE, FAKE, None, FAKE, wsm, 0) == moe.MOE_ERR_INVALID_ARG
    # sizes of the tiled scales equal those of the row-major ones
    k3 = _dims(H=7168, L=3584, E=896, k=16, I=3072, routed=routed)
    st, gu, dn = moe.moe_mx_tiled_scales_size(k3)
    assert st == moe.MOE_OK and gu == 896 * 3072 * 3584 // 16 and dn == 896 * 3584 * 3072 // 32
    assert moe.moe_mx_tiled_scales_size(_dims())[0] == moe.MOE_ERR_UNSUPPORTED
    assert moe.moe_mx_tile_scales(k3, FAKE, None, FAKE, FAKE, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_mx_tile_scales(k3, FAKE, FAKE, FAKE, FAKE + 4, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    # the stand-alone quantisers
    for q in (moe.moe_mx8_quantize, moe.moe_mx4_quantize):
        assert q(FAKE, 4, 48, FAKE, FAKE, 0) == moe.MOE_ERR_INVALID_ARG   # K % 32
        assert q(FAKE + 8, 4, 64, FAKE, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
        assert q(None, 4, 64, FAKE, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
        assert q(None, 0, 64, None, None, 0) == moe.MOE_OK               # nothing to do


def test_gather_rows_validates_on_the_host():
    """moe_gather_rows checks its arguments before any launch."""
    assert moe.moe_gather_rows(FAKE, 4, 32, FAKE, 0, FAKE, 0) == moe.MOE_OK            # nothing to do
    assert moe.moe_gather_rows(None, 0, 32, None, 0, None, 0) == moe.MOE_OK
    assert moe.moe_gather_rows(FAKE, 4, 24, FAKE, 2, FAKE, 0) == moe.MOE_ERR_INVALID_ARG  # row not 16-byte multiple
    assert moe.moe_gather_rows(FAKE, 4, 0, FAKE, 2, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_gather_rows(FAKE, 4, 32, FAKE, -1, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_gather_rows(FAKE, -1, 32, FAKE, 2, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_gather_rows(FAKE, 4, 32, None, 2, FAKE, 0) == moe.MOE_ERR_INVALID_ARG   # no index array
    assert moe.moe_gather_rows(FAKE + 8, 4, 32, FAKE, 2, FAKE, 0) == moe.MOE_ERR_INVALID_ARG  # misaligned


def test_structs_keep_their_tensors_alive():
    """make_weights / make_aux / make_grads hold the tensors whose addresses
    they carry, so a tensor built for the call is not freed (and its memory
    reused) while the struct is in use."""
    import gc
    import weakref

    import torch

    for make, field in ((moe.make_weights, "Sgv_tiled"), (moe.make_aux, "u"), (moe.make_grads, "dx")):
        t = torch.zeros(4)
        ref = weakref.ref(t)
        s = make(**{field: t})
        del t
        gc.collect()
        assert ref() is not None
        del s
        gc.collect()
        assert ref() is None


@pytest.mark.parametrize("name", sorted(gen.CONFIGS))
def test_every_workload_is_valid_and_supported(name):
    """Every workload of gen/configs.py passes the library's host-side dims
    rules (valid and implemented), so its workspace size is positive; the
    block-scaled ones also size their tiled weight scales."""
    cfg = gen.CONFIGS[name]
    d = moe.Dims(T=cfg.T, H=cfg.H, L=cfg.L, E=cfg.E, k=cfg.k, I=cfg.I, S=cfg.S, Is=cfg.Is, act=cfg.act,
                 routed=cfg.routed, y_out="f32", situ_c=cfg.situ_c, rms_eps=cfg.rms_eps)
    assert moe.moe_workspace_size(d) > 0
    if cfg.routed in moe.BLOCK_SCALED:
        st, gu, dn = moe.moe_mx_tiled_scales_size(d)
        assert st == moe.MOE_OK and gu == cfg.E * cfg.I * cfg.L // 16 and dn == cfg.E * cfg.L * cfg.I // 32
