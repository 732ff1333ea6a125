"""The device half of the input generator writes exactly the bits of the host
half, so the oracle (host) and the kernels (device) see the same inputs."""
import numpy as np
import pytest
import torch

import gen

pytestmark = pytest.mark.gpu


def test_device_generator_matches_host():
    cfg = gen.CONFIGS["mid"].with_(T=64)
    w = gen.device_layer(cfg, "cuda")
    for name in ("x", "Wr", "Wdown", "Wsg"):
        t = w[name].view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(t, gen.host_tensor(cfg, name) if name != "x" else gen.host_rows(cfg, "x", range(64)))
    for e in (0, 77, cfg.E - 1):
        assert np.array_equal(w["Wg"][e].view(torch.int16).cpu().numpy().view(np.uint16), gen.host_expert(cfg, "Wg", e))
        assert np.array_equal(w["Wo"][e].view(torch.int16).cpu().numpy().view(np.uint16), gen.host_expert(cfg, "Wo", e))


def test_device_generator_fp32_and_mxfp4():
    tiny = gen.CONFIGS["tiny"]
    w = gen.device_layer(tiny, "cuda")
    assert np.array_equal(w["Wv"].cpu().numpy()[3], gen.host_expert(tiny, "Wv", 3))
    cfg = gen.CONFIGS["mxfp4-small"].with_(T=16)
    w = gen.device_layer(cfg, "cuda")
    for name, sname in (("Wg", "Sg"), ("Wo", "So")):
        for e in (0, 5, cfg.E - 1):
            codes, scales = gen.host_expert(cfg, name, e)
            assert np.array_equal(w[name][e].cpu().numpy(), codes)
            assert np.array_equal(w[sname][e].cpu().numpy(), scales)
