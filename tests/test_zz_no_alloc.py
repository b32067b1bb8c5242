"""moe_permute_noalloc: the permutation for callers that cannot provide a
device workspace (their device memory is planned by another component, or
they own no device allocator), with its scratch in the library's built-in
device array.  Its results must equal moe_permute's (index maps,
probabilities and quantised bytes: bit-exact) on consecutive calls, the
second one overwriting the array the first one used.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process
(the first call performs the per-device set-up)."""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import get_config, make_inputs


def _buffers(torch, cfg, rows_cap, lib):
    dev = "cuda"
    sb = lib.moe_mx_scale_bytes
    T, H, E, k = cfg.T, cfg.H, cfg.E, cfg.k
    return {
        "split": torch.full((E,), -7, dtype=torch.int32, device=dev),
        "offs": torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
        "r2s": torch.full((rows_cap,), -7, dtype=torch.int32, device=dev),
        "s2r": torch.full((T * k,), -7, dtype=torch.int32, device=dev),
        "pp": torch.full((rows_cap,), -7.0, dtype=torch.float32, device=dev),
        "xq": torch.full((rows_cap * H,), 0x5A, dtype=torch.uint8, device=dev),
        "xsf": torch.full((sb(1, rows_cap, H),), 0x5A, dtype=torch.uint8, device=dev),
        "xc": torch.full((H * rows_cap,), 0x5A, dtype=torch.uint8, device=dev),
        "xcsf": torch.full((sb(1, H, rows_cap),), 0x5A, dtype=torch.uint8, device=dev),
    }


def _args(b):
    return (b["split"].data_ptr(), b["offs"].data_ptr(), b["r2s"].data_ptr(), b["s2r"].data_ptr(),
            b["pp"].data_ptr(), b["xq"].data_ptr(), b["xsf"].data_ptr(), b["xc"].data_ptr(),
            b["xcsf"].data_ptr())


@pytest.mark.gpu
def test_permute_noalloc_matches_workspace_entry_point():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mxfp8_grouped_gemm_x32_b200 import lib

    cases = [get_config("tiny", T=384, E=6, k=2),
             get_config("qwen3_30b_ragged", T=512, H=256, I=256, E=128, k=8)]
    for seed, cfg in enumerate(cases, start=1):
        inp = make_inputs(cfg, seed=seed, weights=False, grad=False)
        x = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16).cuda()
        idx = torch.from_numpy(inp["topk_idx"]).cuda()
        prob = torch.from_numpy(inp["topk_prob"]).cuda()
        rows_cap = lib.moe_padded_rows(cfg.T, cfg.k, cfg.E)
        ws_bytes = lib.moe_workspace_size(lib.MOE_OP_PERMUTE, cfg.T, cfg.k, cfg.E, cfg.H, cfg.I)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        ref = _buffers(torch, cfg, rows_cap, lib)
        got = _buffers(torch, cfg, rows_cap, lib)
        lib.moe_permute(x.data_ptr(), idx.data_ptr(), prob.data_ptr(), cfg.T, cfg.H, cfg.k, cfg.E, rows_cap,
                        *_args(ref), ws.data_ptr(), ws_bytes, 0)
        lib.moe_permute_noalloc(x.data_ptr(), idx.data_ptr(), prob.data_ptr(), cfg.T, cfg.H, cfg.k, cfg.E,
                                rows_cap, *_args(got), 0)
        torch.cuda.synchronize()
        assert lib.moe_get_device_status(0) == 0
        for key in ref:
            assert torch.equal(ref[key], got[key]), (cfg.name, key)
        # the histogram scratch really was used: groups are 128-aligned and complete
        offs = got["offs"].cpu().numpy()
        assert offs[0] == 0 and np.all(offs % 128 == 0)
        assert got["split"].sum().item() == cfg.T * cfg.k


def test_permute_noalloc_rejects_problems_beyond_its_scratch():
    """Checked on the host before anything is launched (no device needed)."""
    from mxfp8_grouped_gemm_x32_b200 import lib
    T, k, E, H = 262144, 8, 256, 256          # ceil(T*k/1024) * E * 4 bytes > 256 KB
    rows_cap = lib.moe_padded_rows(T, k, E)
    fake = 1 << 20                             # aligned, never dereferenced
    code = lib._lib.moe_permute_noalloc(fake, fake, fake, T, H, k, E, rows_cap, fake, fake, fake, fake,
                                        fake, fake, fake, 0, 0, None)
    assert code == 8, lib.status_string(code)  # MOE_ERR_TOO_LARGE
    assert "scratch" in lib.status_string(code)
