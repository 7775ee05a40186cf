"""Run one kernel of the library a few times on a seeded synthetic case, for
profiling it (for example under ncu with a kernel filter and a launch skip):

    python -m selective_state_space_40_b200.profile_cases CASE [REPEATS]

CASE is one of: scan130m (selective scan forward, 130M-class layer),
scan130m_reg (the same with the register-prefetch engine), scan2p8b (the
2.8B-class layer), scanlong (the long-context fp32 layer, sequence split),
scanlong_b1_L16k (its first 16384 tokens: a small case of the same kernels),
conv130m (the same with the causal conv front-end, width 4), decode (one
state update at b256 d5120 N16), bwd130m_b4 (training forward with saved
states, then the backward, 130M-class layer with 4 batch rows), ssd2p7b_b2
(Mamba-2 SSD layer, 2.7B-class with 2 batch rows), ssddec_b64 (its one-token
state update for 64 sequences), ssdcb2p7b (the per-chunk
C B^T of that layer on the tcgen05 tensor cores, 4 batch rows). Each kernel
of the case runs REPEATS times (default 3).
"""
from __future__ import annotations

import sys

import torch

from . import binding as mb
from . import synthetic as syn


def _scan(reps, conv=False, w=syn.M130, plan=None):
    g = {k: v.cuda() for k, v in syn.scan_inputs(w).items()}
    y = torch.empty(w.batch, w.dim, w.seqlen, device="cuda")
    last = torch.empty(w.batch, w.dim, w.dstate, device="cuda")
    cp = {k: v.cuda() for k, v in syn.conv_params(w, 4).items()} if conv else None
    for _ in range(reps):
        if conv:
            mb.conv_scan_fwd(g["u"], cp["conv_w"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                             g["delta_bias"], True, conv_b=cp["conv_b"], y=y, last_state=last)
        else:
            mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                        y=y, last_state=last, plan=plan)


def _decode(reps):
    w = syn.DECODE
    p = {k: v.cuda() for k, v in syn.decode_params(w).items()}
    s = {k: v.cuda() for k, v in syn.decode_step_inputs(w, 0).items()}
    state = p["state0"].clone()
    y = torch.empty(w.batch, w.dim, device="cuda")
    for _ in range(reps):
        mb.state_update(state, s["x"], s["delta"], p["A"], s["B"], s["C"], p["D"], s["z"], p["delta_bias"], True,
                        y=y)


def _bwd(reps):
    w = syn.scaled(syn.M130, batch=4)
    g = {k: v.cuda() for k, v in syn.scan_inputs(w).items()}
    dout = torch.randn(w.batch, w.dim, w.seqlen, generator=torch.Generator().manual_seed(1)).cuda()
    for _ in range(reps):
        _, _, ck = mb.scan_fwd_train(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                     True)
        mb.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True, dout,
                    ckpt=ck)


def _ssd(reps):
    w = syn.SsdWorkload("profile", 2, 2048, 80, 64, 128, 1)
    g = {k: v.cuda() for k, v in syn.ssd_inputs(w).items()}
    for _ in range(reps):
        mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True, return_final_state=False)


def _ssd_decode(reps):
    # one-token steps of the 2.7B-class layer for 64 sequences: fp32 state [64, 80, 64, 128]
    w = syn.SsdWorkload("decode", 64, 1, 80, 64, 128, 1)
    par = {k: v.cuda() for k, v in syn.ssd_inputs(w).items()}
    gen = torch.Generator().manual_seed(11)
    state = (0.1 * torch.randn(64, 80, 64, 128, generator=gen)).cuda()
    x = torch.randn(64, 80, 64, generator=gen).to(torch.bfloat16).cuda()
    dt = torch.randn(64, 80, generator=gen).to(torch.bfloat16).cuda()
    B = torch.randn(64, 1, 128, generator=gen).to(torch.bfloat16).cuda()
    C = torch.randn(64, 1, 128, generator=gen).to(torch.bfloat16).cuda()
    for _ in range(reps):
        mb.ssd_state_update(state, x, dt, par["A"], B, C, par["D"], par["dt_bias"], True)


def _ssd_cb(reps):
    w = syn.SSD_2P7B
    g = {k: v.cuda() for k, v in syn.ssd_inputs(w).items()}
    cb = torch.empty(w.batch, w.ngroups, (w.seqlen + 31) // 32, 32, 32, device="cuda")
    for _ in range(reps):
        mb.ssd_chunk_cb(g["B"], g["C"], cb=cb)


CASES = {
    "scan130m": lambda r: _scan(r),
    "scan130m_reg": lambda r: _scan(r, plan=(4, 1, 0, mb.MS_ENGINE_REGISTER)),
    "scan2p8b": lambda r: _scan(r, w=syn.M2P8),
    "scanlong": lambda r: _scan(r, w=syn.LONG),
    "scanlong_b1_L16k": lambda r: _scan(r, w=syn.scaled(syn.LONG, seqlen=16384)),
    "conv130m": lambda r: _scan(r, conv=True),
    "decode": _decode,
    "bwd130m_b4": _bwd,
    "ssd2p7b_b2": _ssd,
    "ssddec_b64": _ssd_decode,
    "ssdcb2p7b": _ssd_cb,
}


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    if not argv or argv[0] not in CASES:
        print(__doc__)
        return 2
    reps = int(argv[1]) if len(argv) > 1 else 3
    torch.cuda.set_device(0)
    CASES[argv[0]](reps)
    torch.cuda.synchronize()
    print("ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
