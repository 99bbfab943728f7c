"""The exchange plumbing between real ranks, on the CPU: two processes over gloo.

Each rank builds its own wire with the oracle (no GPU here), the module's collective helpers move
it between the processes, and the oracle reduces what arrived.  For every scheme the result on
every rank must be bitwise the single-process result over all ranks' partial sums:

  allgather       the stacked wire, then the P-rank reduction of all rows
  reduce_scatter  row blocks all-to-all, the P-rank reduction of the own block, then the rows
                  all-gathered
  two-step        reduce_scatter's first step, then each reducer's block quantized with its own
                  step-2 grid, all-gathered and dequantized block by block

This checks the order and layout of the gathered and scattered shards, which the one-GPU tests
cannot see.
"""
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_WORKER = r'''
import datetime, os, sys
sys.path.insert(0, os.environ["HQ_ROOT"])
import numpy as np
import torch
import torch.distributed as dist
import oracle
import synth
from bit_tensor_activation_b200.exchange import allgather_rows, allgather_stack, alltoall_blocks

rank, port = int(sys.argv[1]), sys.argv[2]
dist.init_process_group("gloo", init_method="tcp://127.0.0.1:" + port, rank=rank, world_size=2,
                        timeout=datetime.timedelta(seconds=60))
o = oracle.get()
cfg = synth.CONFIGS["pr1"].with_(T=24)          # P = 2 ranks, H = 256, k = 8
P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
Tb = T // P
cs, _ = synth.colscale(cfg)
cal = [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T, cs=cs) for b in range(cfg.calib_batches)]
emin, emax = o.calibrate_batches(cal, cfg.beta)
sel = o.select_topk(emin, emax, k)               # what every rank holds after the one statistics exchange
keep, rest, scale, inv, zero = sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"]
x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)    # [P, T, H]; this process plays rank `rank`
codes_all, side_all = o.quantize_pack(x, keep, rest, inv, zero)
ref = o.dequant_reduce(codes_all, side_all, H, keep, rest, scale, zero)

def t32(a): return torch.from_numpy(np.ascontiguousarray(a).view(np.int32))
def t16(a): return torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
def n32(t): return t.numpy().view(np.uint32)
def n16(t): return t.numpy().view(np.uint16)

# allgather: this rank's wire, gathered in rank order, reduced over all rows
c, s = o.quantize_pack(x[rank:rank + 1], keep, rest, inv[rank:rank + 1], zero[rank:rank + 1])
cg, sg = allgather_stack(t32(c)), allgather_stack(t16(s))
assert np.array_equal(n32(cg), codes_all) and np.array_equal(n16(sg), side_all), "gathered wire"
out = o.dequant_reduce(n32(cg), n16(sg), H, keep, rest, scale, zero)
assert np.array_equal(out, ref), "allgather result"

# reduce_scatter: row blocks of this rank's partial sum (all with this rank's grid) to their owners
xb = x[rank].reshape(P, Tb, H)
cb, sb = o.quantize_pack(xb, keep, rest, np.repeat(inv[rank:rank + 1], P, 0), np.repeat(zero[rank:rank + 1], P, 0))
cr, sr = alltoall_blocks(t32(cb)), alltoall_blocks(t16(sb))
mine = slice(rank * Tb, (rank + 1) * Tb)
assert np.array_equal(n32(cr), codes_all[:, mine]), "received code blocks"
assert np.array_equal(n16(sr), side_all[:, :, mine]), "received side blocks"
blk = o.dequant_reduce(n32(cr), n16(sr), H, keep, rest, scale, zero)
full = allgather_rows(t16(blk))
assert np.array_equal(n16(full), ref), "reduce_scatter result"

# two-step: step-2 grids of the two reducers from their reduced calibration blocks, one kept set
k2 = 16
e2min = np.zeros((P, H), np.float32)
e2max = np.zeros((P, H), np.float32)
for b, xc in enumerate(cal):
    cc, sc = o.quantize_pack(xc, keep, rest, inv, zero)
    red = o.dequant_reduce(cc, sc, H, keep, rest, scale, zero)
    tb = xc.shape[1] // P
    for j in range(P):
        mn, mx = o.calibrate(red[None, j * tb:(j + 1) * tb], cfg.beta, b == 0, e2min[j:j + 1], e2max[j:j + 1])
        e2min[j], e2max[j] = mn[0], mx[0]
p2 = o.select_topk(e2min, e2max, k2)
c2, s2 = o.quantize_pack(blk[None], p2["keep_idx"], p2["rest_idx"], p2["inv_scale"][rank:rank + 1],
                         p2["zero"][rank:rank + 1])
c2g, s2g = allgather_stack(t32(c2)), allgather_stack(t16(s2))
got = np.concatenate([o.dequant_reduce(n32(c2g)[b:b + 1], n16(s2g)[b:b + 1], H, p2["keep_idx"], p2["rest_idx"],
                                       p2["scale"][b:b + 1], p2["zero"][b:b + 1]) for b in range(P)])
want = []
for j in range(P):
    cj, sj = o.quantize_pack(ref[None, j * Tb:(j + 1) * Tb], p2["keep_idx"], p2["rest_idx"], p2["inv_scale"][j:j + 1],
                             p2["zero"][j:j + 1])
    want.append(o.dequant_reduce(cj, sj, H, p2["keep_idx"], p2["rest_idx"], p2["scale"][j:j + 1], p2["zero"][j:j + 1]))
assert np.array_equal(got, np.concatenate(want)), "two-step result"
print("RANK_OK", rank, flush=True)
dist.destroy_process_group()
'''


def test_exchange_schemes_gloo_world2():
    port = str(_free_port())
    env = dict(os.environ, HQ_ROOT=ROOT, OMP_NUM_THREADS="1")
    procs = [subprocess.Popen(["timeout", "-k", "10", "180", sys.executable, "-c", _WORKER, str(r), port],
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True, env=env)
             for r in range(2)]
    outs = [p.communicate() for p in procs]
    for p, (out, err) in zip(procs, outs):
        assert p.returncode == 0, err[-3000:]
    assert sorted(l for o, _ in outs for l in o.splitlines() if l.startswith("RANK_OK")) == ["RANK_OK 0", "RANK_OK 1"]
