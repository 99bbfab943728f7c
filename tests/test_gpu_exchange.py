"""The exchange module's kernel calls on one GPU, against the oracle.

P ranks are played one after another on one GPU (a loopback): every rank's ``pack`` runs, the test
moves the buffers the way the collective would (concatenation for an all-gather, block
transposition for an all-to-all), and every rank's reduction runs on what it would have received.
No kernel waits for another rank.  The real collectives are exercised by a one-rank NCCL group
here and by the two-process gloo test on the CPU.
"""
import datetime
import socket

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import oracle  # noqa: E402
from bit_tensor_activation_b200 import exchange as ex  # noqa: E402
from gpu_helpers import DEV, assert_no_device_error, assert_same, to_dev_u16, u16  # noqa: E402


def _setup(cfg):
    o = oracle.get()
    cs, _ = synth.colscale(cfg)
    cal = [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T, cs=cs) for b in range(cfg.calib_batches)]
    emin, emax = o.calibrate_batches(cal, cfg.beta)
    sel = o.select_topk(emin, emax, cfg.k)
    x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    codes, side = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    ref = o.dequant_reduce(codes, side, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
    params = ex.HybridParams(**{n: torch.from_numpy(sel[n]).to(DEV)
                                for n in ("keep_idx", "rest_idx", "scale", "inv_scale", "zero")})
    return o, cal, sel, x, ref, params


CFG = synth.CONFIGS["decode"].with_(T=64)   # P = 4 ranks, H = 4096, k = 64


def test_allgather_loopback():
    o, cal, sel, x, ref, params = _setup(CFG)
    xd = to_dev_u16(x)
    ranks = [ex.HybridAllReduce(params, CFG.T, r, "allgather") for r in range(CFG.P)]
    wires = [ar.pack(xd[r].view(torch.bfloat16)) for r, ar in enumerate(ranks)]
    codes_all = torch.cat([c for c, _ in wires])
    side_all = torch.cat([s for _, s in wires])
    for ar in ranks:
        assert_same(u16(ar.reduce_block(codes_all, side_all)), ref, f"rank {ar.rank}")
    assert_no_device_error()


def test_reduce_scatter_loopback():
    o, cal, sel, x, ref, params = _setup(CFG)
    P, Tb = CFG.P, CFG.T // CFG.P
    xd = to_dev_u16(x)
    ranks = [ex.HybridAllReduce(params, CFG.T, r, "reduce_scatter") for r in range(P)]
    sent = [ar.pack(xd[r].view(torch.bfloat16)) for r, ar in enumerate(ranks)]
    for j, ar in enumerate(ranks):  # rank j receives block j of every rank's wire
        codes_j = torch.stack([c[j] for c, _ in sent])
        side_j = torch.stack([s[j] for _, s in sent])
        assert_same(u16(ar.reduce_block(codes_j, side_j)), ref[j * Tb:(j + 1) * Tb], f"rank {j}'s block")
    assert_no_device_error()


def _oracle_step_two(o, cal, sel, ref, cfg, k2):
    """Step-2 grids and the two-step output composed from oracle calls."""
    P, H = cfg.P, cfg.H
    e2min = np.zeros((P, H), np.float32)
    e2max = np.zeros((P, H), np.float32)
    for b, xc in enumerate(cal):
        cc, sc = o.quantize_pack(xc, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
        red = o.dequant_reduce(cc, sc, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
        tb = xc.shape[1] // P
        for j in range(P):
            mn, mx = o.calibrate(red[None, j * tb:(j + 1) * tb], cfg.beta, b == 0, e2min[j:j + 1], e2max[j:j + 1])
            e2min[j], e2max[j] = mn[0], mx[0]
    p2 = o.select_topk(e2min, e2max, k2)
    Tb = cfg.T // P
    out = []
    for j in range(P):
        cj, sj = o.quantize_pack(ref[None, j * Tb:(j + 1) * Tb], p2["keep_idx"], p2["rest_idx"],
                                 p2["inv_scale"][j:j + 1], p2["zero"][j:j + 1])
        out.append(o.dequant_reduce(cj, sj, H, p2["keep_idx"], p2["rest_idx"], p2["scale"][j:j + 1],
                                    p2["zero"][j:j + 1]))
    return p2, np.concatenate(out)


# k2 = 64: step-2 code rows of 504 words, staged by TMA (one batched dequant launch); k2 = 16:
# rows of 510 words, which TMA cannot stage (the cp.async kernel, one launch per reducer block)
@pytest.mark.parametrize("k2", [64, 16])
def test_two_step_loopback_and_simulated(k2):
    cfg = CFG.with_(calib_T=64)
    o, cal, sel, x, ref, params = _setup(cfg)
    P, T, H, Tb = cfg.P, cfg.T, cfg.H, cfg.T // cfg.P
    p2_ref, want = _oracle_step_two(o, cal, sel, ref, cfg, k2)
    # step-2 grids on the GPU from the same calibration batches
    p2 = ex.step_two_params_simulated([to_dev_u16(c).view(torch.bfloat16) for c in cal], params, k2, cfg.beta)
    for n in ("keep_idx", "rest_idx", "zero"):
        assert_same(getattr(p2, n).cpu().numpy(), p2_ref[n], f"step-2 {n}")
    for n in ("scale", "inv_scale"):
        assert_same(getattr(p2, n).cpu().numpy().view(np.uint32), p2_ref[n].view(np.uint32), f"step-2 {n}")
    xd = to_dev_u16(x).view(torch.bfloat16)
    # loopback through the per-rank phases
    ranks = [ex.TwoStepAllReduce(params, p2, T, r) for r in range(P)]
    sent = [tr.step1.pack(xd[r]) for r, tr in enumerate(ranks)]
    step2 = []
    for j, tr in enumerate(ranks):
        red = tr.step1_reduce(torch.stack([c[j] for c, _ in sent]), torch.stack([s[j] for _, s in sent]))
        assert_same(u16(red), ref[j * Tb:(j + 1) * Tb], f"reducer {j}'s step-1 block")
        c2, s2 = tr.step2_pack(red)
        step2.append((c2.clone(), s2.clone()))
    codes2 = torch.cat([c for c, _ in step2])
    side2 = torch.cat([s for _, s in step2])
    for tr in ranks:
        assert_same(u16(tr.step2_unpack(codes2, side2)), want, f"rank {tr.rank}")
    # the one-GPU simulation, block by block
    k = params.k
    out1 = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    codes = torch.empty((P, T, (H - k) // 8), dtype=torch.int32, device=DEV)
    side = torch.empty((P, k, T), dtype=torch.bfloat16, device=DEV)
    codes2 = torch.empty((P, Tb, (H - k2) // 8), dtype=torch.int32, device=DEV)
    side2 = torch.empty((P, k2, Tb), dtype=torch.bfloat16, device=DEV)
    ex.two_step_simulated(xd, params, p2, out1, out, codes, side, codes2, side2)
    assert_same(u16(out1), ref, "simulated step 1")
    assert_same(u16(out), want, "simulated two-step")
    # the same scheme as one call of the C ABI, in a caller-owned workspace
    import bit_tensor_activation_b200 as hq

    nbytes = hq.hq_two_step_workspace_bytes(P, T, H, k, k2)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    args = (xd, params.keep_idx, params.rest_idx, params.scale, params.inv_scale, params.zero, p2.keep_idx,
            p2.rest_idx, p2.scale, p2.inv_scale, p2.zero)
    out_c = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    hq.hq_two_step_reduce(*args, ws, out_c)
    assert_same(u16(out_c), want, "hq_two_step_reduce, bf16")
    out_f = torch.empty((T, H), dtype=torch.float32, device=DEV)
    hq.hq_two_step_reduce(*args, ws, out_f)
    want_f = []
    for j in range(P):
        cj, sj = o.quantize_pack(ref[None, j * Tb:(j + 1) * Tb], p2_ref["keep_idx"], p2_ref["rest_idx"],
                                 p2_ref["inv_scale"][j:j + 1], p2_ref["zero"][j:j + 1])
        want_f.append(o.dequant_reduce(cj, sj, H, p2_ref["keep_idx"], p2_ref["rest_idx"], p2_ref["scale"][j:j + 1],
                                       p2_ref["zero"][j:j + 1], out_f32=True))
    assert_same(out_f.cpu().numpy().view(np.uint32), np.concatenate(want_f).view(np.uint32), "hq_two_step_reduce, fp32")
    with pytest.raises(hq.HQError):  # a workspace one byte short
        hq.hq_two_step_reduce(*args, ws[:nbytes - 1], out_c)
    assert_no_device_error()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_real_collectives_one_rank_nccl():
    """Every scheme's __call__ through a real one-rank NCCL group (the collectives are then
    copies): the statistics exchange, the selection and the all-reduce, against the oracle."""
    import torch.distributed as dist

    if dist.is_initialized():
        pytest.skip("a process group already exists")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=DEV)
    try:
        cfg = synth.CONFIGS["decode"].with_(P=1, T=32, calib_batches=3)
        o = oracle.get()
        cs, _ = synth.colscale(cfg)
        cal = [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T, cs=cs) for b in range(cfg.calib_batches)]
        emin = torch.empty((1, cfg.H), dtype=torch.float32, device=DEV)
        emax = torch.empty_like(emin)
        for b, c in enumerate(cal):
            ex.calibrate_local(to_dev_u16(c)[0].view(torch.bfloat16), emin, emax, cfg.beta, b == 0)
        params = ex.select_shared(emin, emax, cfg.k)
        e_min, e_max = o.calibrate_batches(cal, cfg.beta)
        sel = o.select_topk(e_min, e_max, cfg.k)
        assert_same(params.keep_idx.cpu().numpy(), sel["keep_idx"], "keep_idx")
        x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
        c, s = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
        ref = o.dequant_reduce(c, s, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
        xd = to_dev_u16(x)[0].view(torch.bfloat16)
        for scheme in ("allgather", "reduce_scatter"):
            out = ex.HybridAllReduce(params, cfg.T, 0, scheme)(xd)
            assert_same(u16(out), ref, scheme)
        assert_no_device_error()
    finally:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------------------------
# The wires read where they lie: one buffer per rank (peer GPUs' memory between real ranks)
# ---------------------------------------------------------------------------------------------
RANKS_CASES = [  # (P, T, H, k): staged side tiles (T % 8 == 0), side read from memory, all 4-bit, 8 ranks
    (4, 64, 4096, 64), (3, 37, 1056, 32), (2, 48, 2048, 0), (8, 40, 4096, 128),
]


@pytest.mark.parametrize("P,T,H,k", RANKS_CASES, ids=[f"P{c[0]}_T{c[1]}_H{c[2]}_k{c[3]}" for c in RANKS_CASES])
def test_dequant_reduce_ranks_equals_stacked(P, T, H, k):
    import bit_tensor_activation_b200 as hq

    cfg = synth.CONFIGS["decode"].with_(name="ranks", P=P, T=T, H=H, k=k, n_out=16, calib_batches=1, calib_T=T)
    o = oracle.get()
    cs, _ = synth.colscale(cfg)
    x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    emin, emax = o.calibrate(x, cfg.beta, True)
    sel = o.select_topk(emin, emax, k)
    codes, side = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    ref = o.dequant_reduce(codes, side, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
    ref_f = o.dequant_reduce(codes, side, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"], out_f32=True)
    prm = {n: torch.from_numpy(sel[n]).to(DEV) for n in ("keep_idx", "rest_idx", "scale", "zero")}
    # every rank's wire in a buffer of its own
    cl = [torch.from_numpy(codes[r].view(np.int32)).to(DEV) for r in range(P)]
    sl = [to_dev_u16(side[r]).view(torch.bfloat16) for r in range(P)]
    out = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    hq.hq_dequant_reduce_ranks(cl, sl, prm["keep_idx"], prm["rest_idx"], prm["scale"], prm["zero"], out)
    out_f = torch.empty((T, H), dtype=torch.float32, device=DEV)
    hq.hq_dequant_reduce_ranks(cl, sl, prm["keep_idx"], prm["rest_idx"], prm["scale"], prm["zero"], out_f)
    stacked = torch.empty_like(out)
    hq.hq_dequant_reduce(torch.stack(cl), torch.stack(sl), prm["keep_idx"], prm["rest_idx"], prm["scale"],
                         prm["zero"], stacked)
    assert_no_device_error()
    assert_same(u16(out), ref, "per-rank buffers, bf16")
    assert_same(u16(stacked), ref, "stacked buffer, bf16")
    assert_same(out_f.cpu().numpy().view(np.uint32), ref_f.view(np.uint32), "per-rank buffers, fp32")


def test_dequant_reduce_ranks_arguments():
    import bit_tensor_activation_b200 as hq

    T, H, k = 8, 1024, 32
    prm = dict(keep_idx=torch.arange(k, dtype=torch.int32, device=DEV),
               rest_idx=torch.arange(k, H, dtype=torch.int32, device=DEV))
    for P, Hh, kk in ((9, H, k), (2, H, k + 8)):   # more than 8 ranks; code rows not a multiple of 16 bytes
        kp = torch.arange(kk, dtype=torch.int32, device=DEV)
        rp = torch.arange(kk, Hh, dtype=torch.int32, device=DEV)
        cl = [torch.zeros((T, (Hh - kk) // 8), dtype=torch.int32, device=DEV) for _ in range(P)]
        sl = [torch.zeros((kk, T), dtype=torch.bfloat16, device=DEV) for _ in range(P)]
        with pytest.raises(hq.HQError):
            hq.hq_dequant_reduce_ranks(cl, sl, kp, rp, torch.ones((P, Hh), device=DEV),
                                       torch.zeros((P, Hh), dtype=torch.uint8, device=DEV),
                                       torch.empty((T, Hh), dtype=torch.bfloat16, device=DEV))
    assert_no_device_error()
    del prm


def test_peer_allreduce_loopback():
    o, cal, sel, x, ref, params = _setup(CFG)
    P, T, H, k = CFG.P, CFG.T, CFG.H, CFG.k
    W = (H - k) // 8
    wires = [(torch.empty((T, W), dtype=torch.int32, device=DEV), torch.empty((k, T), dtype=torch.bfloat16, device=DEV))
             for _ in range(P)]
    ranks = [ex.PeerAllReduce(params, T, r, wires) for r in range(P)]
    xd = to_dev_u16(x)
    for r, pr in enumerate(ranks):
        pr.pack(xd[r].view(torch.bfloat16))
    for pr in ranks:
        assert_same(u16(pr.reduce()), ref, f"rank {pr.rank}")
    assert_no_device_error()
