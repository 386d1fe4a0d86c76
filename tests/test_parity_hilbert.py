"""GPU checks of token reordering: the row gather/scatter kernel against
numpy indexing (byte-exact), and Skip-Softmax prefill in Hilbert order
against the oracle run on the same reordered inputs."""
import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from oracle.hilbert import hilbert_order
from parity_helpers import bf16_host, check_counts, compare_prefill_units, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("shape,dtype", [((6, 300, 64), torch.bfloat16),
                                         ((2, 3, 1000, 128), torch.bfloat16),
                                         ((4, 777, 1), torch.float32),
                                         ((3, 129, 3), torch.float32)])
def test_permute_rows_exact(shape, dtype):
    L = shape[-2]
    g = torch.Generator().manual_seed(L)
    src = torch.randn(shape, generator=g).to(dtype).cuda()
    perm = torch.randperm(L, generator=g).to(torch.int32)
    idx = perm.cuda()
    dst = torch.empty_like(src)
    sk.sskip_permute_rows(src, dst, idx, scatter=False)
    back = torch.empty_like(src)
    sk.sskip_permute_rows(dst, back, idx, scatter=True)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    s = src.cpu()
    assert torch.equal(dst.cpu(), s[..., perm.long(), :])
    assert torch.equal(back.cpu(), s)


def test_permute_rows_flags_a_bad_index():
    src = torch.zeros((2, 64, 64), dtype=torch.bfloat16, device="cuda")
    dst = torch.full_like(src, 7.0)
    idx = torch.arange(64, dtype=torch.int32, device="cuda")
    idx[5] = 64  # out of range: the kernel's bounds check must catch it
    sk.sskip_permute_rows(src, dst, idx, scatter=False)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_ERR_INVALID_ARG
    assert torch.all(dst[:, 5] == 7.0) and torch.all(dst[:, :5] == 0)
    assert sk.sskip_get_status() == sk.SSKIP_OK  # reading clears the word


def small_video(**kw):
    base = dict(synth.VIDEO_DIT_PREFILL.__dict__)
    # A 5 x 16 x 25 grid: enough keys per row that |O| stays below ~1.8, as
    # on the full workload (a smaller grid gives peaked rows with |O| ~ 3,
    # where bf16 rounding of O alone nears the 1e-2 bound); t = 1000 / 2000.
    base.update(name="t", B=1, Hq=2, Hkv=2, L=2000, video_grid=(5, 16, 25), tsf=1000.0)
    base.update(kw)
    return synth.PrefillWorkload(**base)


def reordered_parity(w, x, perm, n_units=None, seed=0):
    dev_perm = torch.from_numpy(perm).cuda()
    q, k, v = to_device(x["q"]), to_device(x["k"]), to_device(x["v"])
    out = sk.prefill_reordered(q, k, v, dev_perm, sm_scale=w.scale,
                               threshold_scale_factor=w.tsf, Br=w.Br, Bc=w.Bc, with_tiles=True)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    xp = {n: np.ascontiguousarray(x[n][:, :, perm]) for n in ("q", "k", "v")}
    if n_units is None:
        units = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.n_q)]
    else:
        rng = np.random.default_rng(seed)
        units = [(int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(i))
                 for i in np.linspace(0, w.n_q - 1, n_units).astype(int)]
    ora = oracle.prefill(xp["q"], xp["k"], xp["v"], causal=False, sm_scale=w.scale, tsf=w.tsf,
                         Br=w.Br, Bc=w.Bc, units=np.array(units, np.int32), want_margin=True)
    # Outputs came back in the original order; compare in the reordered frame.
    g = {"o": bf16_host(out["o"])[:, :, perm], "lse": out["lse"].cpu().numpy()[:, :, perm],
         "tile_state": out["tile_state"].cpu().numpy()}
    compare_prefill_units(w, xp, g, ora, units)
    return out


@pytest.mark.parametrize("Br", [64, 128])
def test_hilbert_prefill_small(Br):
    w = small_video(Br=Br, Bc=Br)
    x = synth.prefill_inputs(w, "lit")
    perm = hilbert_order(*w.video_grid, w.L)
    out = reordered_parity(w, x, perm)
    ora = oracle.prefill(*(np.ascontiguousarray(x[n][:, :, perm]) for n in ("q", "k", "v")),
                         causal=False, sm_scale=w.scale, tsf=w.tsf, Br=w.Br, Bc=w.Bc)
    c = out["counts"].cpu().tolist()
    check_counts(c[0], ora["skipped"], c[1], ora["visited"])


def test_hilbert_prefill_video_full_size():
    w = synth.VIDEO_DIT_PREFILL
    x = synth.prefill_inputs(w, "lit")
    perm = sk.sskip_hilbert3d_order(*w.video_grid, w.L)
    out = reordered_parity(w, x, perm, n_units=10, seed=3)
    c = out["counts"].cpu().tolist()
    assert c[1] == w.B * w.Hq * w.n_q * w.n_k
