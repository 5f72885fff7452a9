"""Extensions beyond the core path, against the oracle:
  - score matrices in place of W (review: the solver plugs into layer-wise
    pruning such as Wanda, SparseGPT, ALPS, which hand it importance scores);
  - the monotonicity safeguard (review: "Assumptions & free parameters",
    Assumption 1; referee comment 2).
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import NEAR_TIE, block_bits, mask_to_np, max_inverted_gap, record, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import sparse_mask_search_b200 as tsl  # noqa: E402


@pytest.mark.parametrize("M,N", [(8, 4), (16, 8), (32, 16), (64, 32)])
def test_wanda_style_scores(M, N):
    rows, cols = 2 * M, 6 * M
    _, W = synth.make_matrix(rows, cols, "f32", "normal", 0.02, seed=M)
    xnorm = 0.5 + synth.rng(100 + M).random(cols).astype(np.float32)       # input feature norms
    scores = (np.abs(W) * xnorm[None, :]).astype(np.float32)
    sd = to_device(scores, "f32")
    m = mask_to_np(tsl.tsenor_mask_scores(sd, N, M, 20.0, 200, 4))
    assert (m == mask_to_np(tsl.tsenor_mask(sd, N, M, 20.0, 200, 4))).all()
    m_ref, _, _ = oracle.mask(scores, N, M, 20.0, 200, 4)
    bg, br = block_bits(m, cols, M), block_bits(m_ref, cols, M)
    assert (bg.sum(axis=3) == N).all() and (bg.sum(axis=2) == N).all()
    assert (bg == br).all()


@pytest.mark.parametrize("M,N,dtype", [(4, 2, "f32"), (8, 4, "bf16"), (16, 5, "bf16"), (32, 16, "bf16"),
                                       (64, 32, "bf16")])
def test_safeguard_matches_oracle(M, N, dtype):
    rows, cols = 2 * M, 9 * M
    stor, W = synth.make_matrix(rows, cols, dtype, "t3_outlier_cols", 0.02, seed=7 + M)
    Wd = to_device(stor, dtype)
    tau, iters, sweeps = 20.0, 150, 4
    new = mask_to_np(tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps))
    opt, best = oracle.opt(W, N, M, want_mask=True)
    prev_cases = [best, new, np.full_like(new, 0xFFFFFFFF)]
    for prev in prev_cases:
        kept = torch.zeros(1, dtype=torch.int64, device="cuda")
        prev_d = torch.from_numpy(np.ascontiguousarray(prev).view(np.int32)).cuda()
        out = mask_to_np(tsl.tsenor_mask_safeguard(Wd, prev_d, N, M, tau, iters, sweeps, kept=kept))
        ref, kept_ref = oracle.safeguard(W, prev, new, N, M)
        assert (out == ref).all()
        assert int(kept.item()) == kept_ref
    # with the optimum as the previous mask the result is optimal everywhere
    kept = torch.zeros(1, dtype=torch.int64, device="cuda")
    out = tsl.tsenor_mask_safeguard(Wd, torch.from_numpy(best.view(np.int32)).cuda(), N, M, tau, iters, sweeps,
                                    kept=kept)
    np.testing.assert_allclose(tsl.tsenor_objective(Wd, out, N, M).cpu().numpy(), opt, rtol=1e-12)


@pytest.mark.parametrize("rows,cols,M,N,dtype", [(100, 70, 32, 16, "bf16"), (50, 37, 8, 4, "f32"),
                                                 (17, 48, 16, 8, "bf16"), (64, 64, 16, 8, "bf16"),
                                                 (9, 130, 64, 32, "bf16"), (6, 10, 4, 2, "f32")])
def test_padded_shapes(rows, cols, M, N, dtype):
    """Zero-pad to multiples of M, solve, crop (the padding reading of the review's block partition)."""
    stor, W = synth.make_matrix(rows, cols, dtype, "normal", 0.02, seed=rows + cols)
    m = mask_to_np(tsl.tsenor_mask_padded(to_device(stor, dtype), N, M, 20.0, 150, 4))
    rp, cp = -(-rows // M) * M, -(-cols // M) * M
    Wp = np.zeros((rp, cp), np.float32)
    Wp[:rows, :cols] = W
    m_ref_p, keys_ref, _ = oracle.mask(Wp, N, M, 20.0, 150, 4, want_keys=True)
    ref_bits = oracle.unpack(m_ref_p, cp)[:rows, :cols]
    bits = oracle.unpack(m, cols)
    assert m.shape == (rows, (cols + 31) // 32)
    assert (oracle.unpack(m, m.shape[1] * 32)[:, cols:] == 0).all()       # padding bits are 0
    # the cropped mask of the padded solve, on the GPU, bit for bit
    stor_p = np.zeros((rp, cp), dtype=np.asarray(stor).dtype)
    stor_p[:rows, :cols] = stor
    Wpd = to_device(stor_p, dtype)
    full = mask_to_np(tsl.tsenor_mask(Wpd, N, M, 20.0, 150, 4))
    assert (oracle.unpack(full, cp)[:rows, :cols] == bits).all()
    # against the oracle: blocks identical except where the oracle's keys hold
    # a near-tie that the fp32 plan orders the other way (zero padding makes
    # many entries equal up to rounding)
    gpu_bits_p = oracle.unpack(full, cp)
    same = (oracle.blocks_view(gpu_bits_p, M) == oracle.blocks_view(oracle.unpack(m_ref_p, cp), M)).all(axis=(2, 3))
    if not same.all():
        plan = tsl.tsenor_plan(Wpd, N, M, 20.0, 150).cpu().numpy()
        Pg, Pr, A = oracle.blocks_view(plan, M), oracle.blocks_view(keys_ref, M), oracle.blocks_view(np.abs(Wp), M)
        for r, c in zip(*np.nonzero(~same)):
            assert max_inverted_gap(Pr[r, c], Pg[r, c], A[r, c]) <= NEAR_TIE, (r, c)
    record(f"padded-{rows}x{cols}-{N}of{M}", {"blocks": int(same.size), "identical": float(same.mean())})
    # every row / column of a block keeps at most N (exactly N where the block is full)
    full_r, full_c = rows // M * M, cols // M * M
    if full_r and full_c:
        fb = oracle.blocks_view(bits[:full_r, :full_c], M)
        assert (fb.sum(axis=3) == N).all() and (fb.sum(axis=2) == N).all()
    for r0 in range(0, rows, M):
        for c0 in range(0, cols, M):
            blk = bits[r0:r0 + M, c0:c0 + M]
            assert (blk.sum(axis=1) <= N).all() and (blk.sum(axis=0) <= N).all()


@pytest.mark.parametrize("rows,cols,M,N,dtype", [(4096, 1024, 32, 16, "bf16"), (1000 // 8 * 8, 96, 8, 4, "f32"),
                                                 (64, 64, 16, 8, "bf16"), (8 * 64, 128, 64, 32, "bf16"),
                                                 (36, 40, 4, 2, "f32"),
                                                 # 17 MB and 32 MB of W: two and four chunks, the last one shorter
                                                 (4192, 2048, 32, 16, "bf16"), (4096, 2048, 8, 4, "f32")])
def test_host_pipeline_matches_device_call(rows, cols, M, N, dtype):
    """tsenor_mask_host (row chunks of ~8 MB pipelined through two device slots) gives tsenor_mask's mask."""
    stor, W = synth.make_matrix(rows, cols, dtype, "t3_outlier_cols", 0.02, seed=rows + M)
    Wd = to_device(stor, dtype)
    ref = tsl.tsenor_mask(Wd, N, M, 20.0, 120, 4).cpu()
    Wh = Wd.cpu().pin_memory()
    side = torch.cuda.Stream()
    out = tsl.tsenor_mask_host(Wh, N, M, 20.0, 120, 4, stream=side)
    side.synchronize()
    assert torch.equal(out, ref)
    # pageable buffers work too
    out2 = tsl.tsenor_mask_host(Wd.cpu(), N, M, 20.0, 120, 4, out=torch.zeros_like(ref))
    torch.cuda.current_stream().synchronize()
    assert torch.equal(out2, ref)


def test_host_pipeline_from_two_threads():
    """Each host thread keeps its own pipeline streams and events: two threads
    calling tsenor_mask_host at the same time, several times each on their own
    streams, all get tsenor_mask's mask."""
    import threading
    stor, W = synth.make_matrix(4096, 2048, "bf16", "t3_outlier_cols", 0.02, seed=11)
    Wd = to_device(stor, "bf16")
    ref = tsl.tsenor_mask(Wd, 16, 32, 20.0, 120, 4).cpu()
    Wh = Wd.cpu().pin_memory()
    outs, errs = [None, None], []

    def run(k):
        try:
            torch.cuda.set_device(Wd.device)
            s = torch.cuda.Stream()
            got = []
            for _ in range(3):
                got.append(tsl.tsenor_mask_host(Wh, 16, 32, 20.0, 120, 4, stream=s))
            s.synchronize()
            outs[k] = got
        except Exception as e:                      # reported below, in the main thread
            errs.append(e)

    threads = [threading.Thread(target=run, args=(k,)) for k in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errs, errs
    for got in outs:
        for o in got:
            assert torch.equal(o, ref)


@pytest.mark.parametrize("M,N", [(8, 4), (16, 8), (32, 16), (64, 32)])
def test_offsets_beyond_int32(M, N):
    """A matrix of more than 2^31 elements (bf16, generated on the device from a
    seeded generator): every block valid, and blocks at the far end of the
    matrix equal to the oracle's."""
    rows, cols = 65536, 32832                                # 2.15e9 elements, cols a multiple of 64
    assert rows * cols > 2 ** 31
    g = torch.Generator(device="cuda")
    g.manual_seed(1234 + M)
    Wd = (0.02 * torch.randn((rows, cols), device="cuda", generator=g)).to(torch.bfloat16)
    tau, iters, sweeps = 20.0, 30, 2
    tsl.tsenor_error_count()
    mask = tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps)
    obj = tsl.tsenor_objective(Wd, mask, N, M)
    assert tsl.tsenor_error_count() == 0
    assert not torch.isnan(obj).any()
    # the last block-row and a block-row across the 2^31-element mark, against the oracle
    for r0 in (rows - M, (2 ** 31 // cols) // M * M):
        sub = Wd[r0:r0 + M].float().cpu().numpy()
        m_ref, keys_ref, _ = oracle.mask(sub, N, M, tau, iters, sweeps, want_keys=True)
        m_gpu = mask[r0:r0 + M].cpu().numpy().view(np.uint32)
        bg, br = block_bits(m_gpu, cols, M), block_bits(m_ref, cols, M)
        assert (bg.sum(axis=3) == N).all() and (bg.sum(axis=2) == N).all()
        same = (bg == br).all(axis=(2, 3)).ravel()
        if not same.all():
            # a differing block must come from a near-tie of the oracle's keys (blocks are
            # independent, so the plan of this block-row alone is the plan of the full solve)
            plan = tsl.tsenor_plan(Wd[r0:r0 + M].contiguous(), N, M, tau, iters).cpu().numpy()
            Pg, Pr = oracle.blocks_view(plan, M), oracle.blocks_view(keys_ref, M)
            A = oracle.blocks_view(np.abs(sub), M)
            for c in np.nonzero(~same)[0]:
                assert max_inverted_gap(Pr[0, c], Pg[0, c], A[0, c]) <= NEAR_TIE, (r0, c)
        assert same.mean() >= 0.999
    del Wd, mask, obj
    torch.cuda.empty_cache()
