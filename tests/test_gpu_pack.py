"""nq_pack_signs on the GPU against the oracle's pack: bit-exact on every word."""
import numpy as np
import pytest
import torch

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import need_gpu, nq

pytestmark = pytest.mark.gpu


def run_pack(latent_np, r, ld_words, ld_latent=None):
    rows = latent_np.shape[0]
    ld_latent = latent_np.shape[1] if ld_latent is None else ld_latent
    buf = np.zeros((rows, ld_latent), dtype=np.float32)
    buf[:, : latent_np.shape[1]] = latent_np
    dev = torch.from_numpy(buf).cuda()
    out = nq().pack_signs(dev[:, :r] if r <= ld_latent else dev, r=r, ld_words=ld_words)
    torch.cuda.synchronize()
    nq().sync_status()
    return out.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("rows,r,ld_words", [(256, 128, 4), (512, 128, 4), (37, 96, 5), (1, 32, 1), (3, 1024, 33),
                                             (1000, 3520, 110), (129, 2240, 72)])
def test_pack_random_bit_exact(rows, r, ld_words):
    need_gpu()
    L = synth.latent_f32(synth.rng_for(101, rows, r), rows, r)
    got = run_pack(L, r, ld_words)
    want = oracle.pack(L, r=r, ld_words=ld_words)
    np.testing.assert_array_equal(got, want)


def test_pack_padded_latent_rows():
    need_gpu()
    rows, r, ld_latent = 70, 64, 100
    L = synth.latent_f32(synth.rng_for(102), rows, ld_latent)
    got = run_pack(L, r, 2, ld_latent=ld_latent)
    want = oracle.pack(L[:, :r].copy(), r=r, ld_words=2)
    np.testing.assert_array_equal(got, want)


def test_pack_edge_values():
    need_gpu()
    vals = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-45, -1e-45, 3.4e38, -3.4e38, 1.0, -1.0],
                    dtype=np.float32)
    rng = np.random.default_rng(5)
    L = rng.choice(vals, size=(64, 256)).astype(np.float32)
    L[3, 5] = np.float32(-0.0)
    got = run_pack(L, 256, 9)
    want = oracle.pack(L, r=256, ld_words=9)
    np.testing.assert_array_equal(got, want)


def test_pack_empty_is_noop():
    need_gpu()
    out = torch.full((0, 4), 7, dtype=torch.int32, device="cuda")
    nq().pack_signs(torch.empty((0, 128), dtype=torch.float32, device="cuda"), r=128, ld_words=4, out=out)
    nq().sync_status()


def test_pack_full_size_70b_gate_u():
    """The largest pack in the workloads: U of the 70B gate projection, 28672 x 3520."""
    need_gpu()
    rows, r = 28672, 3520
    L = synth.latent_f32(synth.rng_for(103), rows, r)
    got = run_pack(L, r, r // 32)
    want = oracle.pack(L, r=r, ld_words=r // 32)
    np.testing.assert_array_equal(got, want)
