"""Every kernel reads and writes only inside the tensors it is given.  Each tensor of a call sits
in the middle of a larger buffer: the margins of inputs hold NaN (a read there would poison the
results), the margins of outputs and of the workspace hold a sentinel (a write there would change
it).  The shapes leave idle lanes, idle warps and whole idle warps of a CTA, ragged time tails and
partial channel tiles.  The results must equal those of the same call on plain tensors bitwise,
and every margin must be intact afterwards.  All accesses stay inside the enlarged buffers, so a
stray access changes values here instead of touching memory the test does not own."""
import math

import pytest
import torch

import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200 import _abi
from selective_state_space_23_b200.inputs import make_inputs, workload

pytestmark = pytest.mark.gpu
DEV = "cuda"
PAD = 4096  # margin elements on each side (a multiple of 16 bytes for every dtype)
SENT = -7.25
IO_CODE = {torch.float32: 0, torch.bfloat16: 1}


class Arena:
    """Places tensors inside NaN- or sentinel-filled buffers and checks the margins later."""

    def __init__(self, guarded):
        self.guarded = guarded
        self.bufs = []

    def _place(self, shape, dtype, fill):
        n = math.prod(shape)
        if not self.guarded:
            return torch.full(shape, fill, dtype=dtype, device=DEV)
        buf = torch.full((2 * PAD + n,), fill, dtype=dtype, device=DEV)
        self.bufs.append((buf, n, fill))
        return buf[PAD:PAD + n].view(shape)

    def inp(self, t):
        if t is None:
            return None
        v = self._place(tuple(t.shape), t.dtype, float("nan"))
        v.copy_(t.to(DEV))
        return v

    def out(self, shape, dtype):
        return self._place(tuple(shape), dtype, SENT)

    def workspace(self, nbytes):
        if nbytes == 0:
            return None
        if not self.guarded:
            return torch.empty(nbytes, dtype=torch.uint8, device=DEV)
        buf = torch.full((2 * PAD + nbytes,), 0xA5, dtype=torch.uint8, device=DEV)
        self.bufs.append((buf, nbytes, 0xA5))
        return buf[PAD:PAD + nbytes]

    def check_margins(self):
        torch.cuda.synchronize()
        for buf, n, fill in self.bufs:
            m = torch.cat([buf[:PAD], buf[PAD + n:]])
            if isinstance(fill, float) and math.isnan(fill):
                assert torch.isnan(m.float()).all(), "an input margin changed"
            else:
                assert (m == fill).all(), "a write landed outside its tensor"


def p(t):
    return 0 if t is None else t.data_ptr()


def inputs(batch, dim, L, N, io, G=1, scalar_a=False, channels_last=False, seed=31):
    w = workload("mamba2p8b_train", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=seed, with_dout=True, with_h0=True, scalar_a=scalar_a)
    if G > 1:
        wg = workload("mamba2p8b_train", batch=batch * G, dim=1, seqlen=L, dstate=N, io_dtype=io)
        xg = make_inputs(wg, seed=seed + 1)
        x["B"] = xg["B"].reshape(batch, G, N, L).contiguous()
        x["C"] = xg["C"].reshape(batch, G, N, L).contiguous()
    if channels_last:
        for k in ("u", "delta", "z", "dout"):
            x[k] = x[k].transpose(1, 2).contiguous()
        for k in ("B", "C"):
            b = x[k] if x[k].dim() == 4 else x[k].unsqueeze(1)
            x[k] = b.permute(0, 3, 1, 2).contiguous()
    return x


def run_fwd(x, guarded, batch, dim, L, N, G, flags, ckpt=True):
    ar = Arena(guarded)
    io = x["u"].dtype
    t = {k: ar.inp(v) for k, v in x.items()}
    xs = tuple(x["u"].shape)
    out = ar.out(xs, io)
    hL = ar.out((batch, dim, N), torch.float32)
    nblk = (L + 15) // 16
    ck = ar.out((batch, dim, nblk, N), torch.float32) if ckpt else None
    lib = _abi.lib()
    nws = int(lib.ssm_scan_fwd_ex_workspace_size(batch, dim, L, N, G, IO_CODE[io], flags))
    ws = ar.workspace(nws)
    rc = lib.ssm_scan_fwd_ex(p(t["u"]), p(t["delta"]), p(t["A"]), p(t["B"]), p(t["C"]), p(t["D"]),
                             p(t["z"]), p(t["dt_bias"]), 1, p(t["h0"]), p(hL), p(out), p(ck), p(ws),
                             nws, batch, dim, L, N, G, IO_CODE[io], flags, 0)
    _abi.check(rc, "ssm_scan_fwd_ex")
    ar.check_margins()
    return [out.clone(), hL.clone()] + ([ck.clone()] if ckpt else [])


def run_bwd(x, guarded, batch, dim, L, N, G, flags, scalar_a=False):
    ar = Arena(guarded)
    io = x["u"].dtype
    t = {k: ar.inp(v) for k, v in x.items()}
    xs = tuple(x["u"].shape)
    bc = tuple(x["B"].shape)
    g = {"du": ar.out(xs, io), "ddelta": ar.out(xs, io), "dz": ar.out(xs, io),
         "dB": ar.out(bc, io), "dC": ar.out(bc, io),
         "dA": ar.out((dim,) if scalar_a else (dim, N), torch.float32),
         "dD": ar.out((dim,), torch.float32), "ddt_bias": ar.out((dim,), torch.float32),
         "dh0": ar.out((batch, dim, N), torch.float32)}
    lib = _abi.lib()
    nws = int(lib.ssm_scan_bwd_ex_workspace_size(batch, dim, L, N, G, IO_CODE[io], 0, flags))
    ws = ar.workspace(nws)
    rc = lib.ssm_scan_bwd_ex(p(t["u"]), p(t["delta"]), p(t["A"]), p(t["B"]), p(t["C"]), p(t["D"]),
                             p(t["z"]), p(t["dt_bias"]), 1, p(t["h0"]), p(t["dout"]), 0, 0,
                             p(g["du"]), p(g["ddelta"]), p(g["dA"]), p(g["dB"]), p(g["dC"]),
                             p(g["dD"]), p(g["dz"]), p(g["ddt_bias"]), p(g["dh0"]), p(ws), nws,
                             batch, dim, L, N, G, IO_CODE[io], flags, 0)
    _abi.check(rc, "ssm_scan_bwd_ex")
    ar.check_margins()
    return [v.clone() for v in g.values()]


def same(a, b):
    for u, v in zip(a, b):
        assert not torch.isnan(u.float()).any(), "NaN in the results"
        assert torch.equal(u, v), "results differ from those of the plain call"


FWD_CASES = {
    # name: (env, batch, dim, L, N, io, G, flags)
    "general_bf16": ({}, 2, 96, 312, 16, torch.bfloat16, 1, 0),
    "general_f32_ragged": ({}, 2, 40, 37, 5, torch.float32, 1, 0),
    "general_wpb4": ({"SSM_FWD_WPB": "4"}, 2, 96, 312, 16, torch.bfloat16, 1, 0),
    "lane": ({"SSM_FWD_KERNEL": "lane"}, 2, 96, 312, 16, torch.bfloat16, 1, 0),
    "time_split": ({"SSM_FWD_SPLIT": "3"}, 1, 40, 300, 16, torch.bfloat16, 1, 0),
    "channels_last": ({}, 2, 96, 312, 16, torch.bfloat16, 1, 8),
    "reverse_zoh": ({}, 2, 96, 200, 16, torch.bfloat16, 1, 2 | 4),
    "grouped": ({}, 2, 64, 200, 16, torch.bfloat16, 2, 0),
    "per_channel_bc": ({}, 2, 24, 120, 16, torch.bfloat16, 24, 0),
    "scalar_decay": ({}, 2, 96, 200, 16, torch.bfloat16, 1, 1),
    "chunked_n64": ({}, 2, 96, 200, 64, torch.bfloat16, 1, 1),
    "chunked_n128_split": ({"SSM_SSD_SPLIT": "3"}, 1, 80, 333, 128, torch.bfloat16, 1, 1),
    "chunked_n64_reverse": ({}, 1, 80, 333, 64, torch.bfloat16, 1, 1 | 2),
    "chunked_n64_zoh": ({}, 1, 80, 333, 64, torch.bfloat16, 1, 1 | 4),
    "slices_f32_n64": ({}, 2, 40, 37, 64, torch.float32, 1, 1),
    "slices_f32_n32_reverse_zoh_grouped": ({}, 2, 64, 120, 32, torch.float32, 2, 1 | 2 | 4),
}


@pytest.mark.parametrize("case", sorted(FWD_CASES))
def test_forward_stays_inside_its_tensors(monkeypatch, case):
    env, batch, dim, L, N, io, G, flags = FWD_CASES[case]
    for k in ("SSM_FWD_KERNEL", "SSM_FWD_WPB", "SSM_FWD_SPLIT", "SSM_SSD_SPLIT"):
        monkeypatch.delenv(k, raising=False)
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    x = inputs(batch, dim, L, N, io, G=G if G < dim else 1, scalar_a=bool(flags & 1),
               channels_last=bool(flags & 8))
    if G == dim:  # B/C per channel: [batch][dim][N][L]
        w = workload("mamba2p8b_train", batch=batch * dim, dim=1, seqlen=L, dstate=N, io_dtype=io)
        xg = make_inputs(w, seed=77)
        x["B"] = xg["B"].reshape(batch, dim, N, L).contiguous()
        x["C"] = xg["C"].reshape(batch, dim, N, L).contiguous()
    ckpt = N <= 16 or (flags & 1)  # the chunked form (scalar decay) writes checkpoints too
    plain = run_fwd(x, False, batch, dim, L, N, G, flags, ckpt)
    guarded = run_fwd(x, True, batch, dim, L, N, G, flags, ckpt)
    same(guarded, plain)


BWD_CASES = {
    "history_w4": ({"SSM_BWD_WPB": "4"}, 2, 96, 312, 16, torch.bfloat16, 1, 0),
    "history_w2": ({"SSM_BWD_WPB": "2"}, 2, 72 + 8, 312, 16, torch.bfloat16, 1, 0),
    "history_f32": ({}, 2, 96, 200, 16, torch.float32, 1, 0),
    "history_split3": ({"SSM_BWD_SPLIT": "3"}, 2, 96, 312, 16, torch.bfloat16, 1, 0),
    "history_split7_f32": ({"SSM_BWD_SPLIT": "7"}, 1, 80, 200, 16, torch.float32, 1, 0),
    "general": ({"SSM_BWD_KERNEL": "pair"}, 2, 96, 312, 16, torch.bfloat16, 1, 0),
    "general_wpb2": ({"SSM_BWD_KERNEL": "pair", "SSM_BWD_WPB": "2"}, 2, 80, 250, 16,
                     torch.bfloat16, 1, 0),
    "general_ragged_f32": ({}, 2, 40, 37, 5, torch.float32, 1, 0),
    "channels_last": ({}, 2, 96, 312, 16, torch.bfloat16, 1, 8),
    "reverse_zoh_grouped": ({}, 2, 64, 200, 16, torch.bfloat16, 2, 2 | 4),
    "per_channel_bc": ({}, 2, 24, 120, 16, torch.bfloat16, 24, 0),
    "scalar_decay": ({}, 2, 96, 200, 16, torch.bfloat16, 1, 1),
    "scalar_decay_state": ({"SSM_SCALAR_BWD": "state"}, 2, 96, 200, 16, torch.bfloat16, 1, 1),
    "scalar_decay_n64_slices": ({"SSM_SCALAR_BWD": "slices"}, 2, 96, 120, 64, torch.bfloat16, 1, 1),
    "scalar_decay_n64_chunked": ({}, 2, 96, 120, 64, torch.bfloat16, 1, 1),
    "scalar_decay_n128_chunked": ({}, 1, 80, 333, 128, torch.bfloat16, 1, 1),
    "scalar_decay_n64_chunked_split": ({"SSM_SSD_BWD_SPLIT": "3"}, 1, 80, 333, 64, torch.bfloat16, 1, 1),
    "scalar_decay_n64_chunked_reverse": ({}, 1, 80, 333, 64, torch.bfloat16, 1, 1 | 2),
    "scalar_decay_n64_chunked_zoh": ({}, 1, 80, 333, 64, torch.bfloat16, 1, 1 | 4),
}


@pytest.mark.parametrize("case", sorted(BWD_CASES))
def test_backward_stays_inside_its_tensors(monkeypatch, case):
    env, batch, dim, L, N, io, G, flags = BWD_CASES[case]
    for k in ("SSM_FWD_KERNEL", "SSM_BWD_KERNEL", "SSM_BWD_WPB", "SSM_BWD_SPLIT", "SSM_SCALAR_BWD",
              "SSM_SSD_BWD_SPLIT"):
        monkeypatch.delenv(k, raising=False)
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    x = inputs(batch, dim, L, N, io, G=G if G < dim else 1, scalar_a=bool(flags & 1),
               channels_last=bool(flags & 8))
    if G == dim:
        w = workload("mamba2p8b_train", batch=batch * dim, dim=1, seqlen=L, dstate=N, io_dtype=io)
        xg = make_inputs(w, seed=78)
        x["B"] = xg["B"].reshape(batch, dim, N, L).contiguous()
        x["C"] = xg["C"].reshape(batch, dim, N, L).contiguous()
    plain = run_bwd(x, False, batch, dim, L, N, G, flags, scalar_a=bool(flags & 1))
    guarded = run_bwd(x, True, batch, dim, L, N, G, flags, scalar_a=bool(flags & 1))
    same(guarded, plain)


DECODE_CASES = {
    # name: (env, batch, dim, N, io, G, flags)
    "streamed": ({}, 7, 384, 16, torch.bfloat16, 1, 0),
    "streamed_grouped": ({}, 5, 384, 16, torch.float32, 3, 0),
    "per_thread": ({"SSM_DECODE_STREAM": "0"}, 7, 96, 16, torch.bfloat16, 1, 0),
    "per_thread_ragged": ({}, 3, 40, 5, torch.float32, 1, 0),
    "per_channel_bc": ({}, 3, 40, 16, torch.bfloat16, 40, 0),
    "scalar_n64": ({}, 3, 40, 64, torch.bfloat16, 1, 1),
    "scalar_n128_grouped_zoh": ({}, 3, 64, 128, torch.float32, 2, 1 | 4),
}


@pytest.mark.parametrize("case", sorted(DECODE_CASES))
def test_decode_stays_inside_its_tensors(monkeypatch, case):
    env, batch, dim, N, io, G, flags = DECODE_CASES[case]
    monkeypatch.delenv("SSM_DECODE_STREAM", raising=False)
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    gen = torch.Generator().manual_seed(9)
    rnd = lambda *s: torch.randn(*s, generator=gen)
    state0 = 0.5 * rnd(batch, dim, N)
    vals = {"x": rnd(batch, dim).to(io), "dt": (0.3 * rnd(batch, dim)).to(io),
            "z": rnd(batch, dim).to(io),
            "A": -torch.rand(*((dim,) if flags & 1 else (dim, N)), generator=gen) * 4 - 0.1,
            "B": rnd(batch, G, N).to(io), "C": rnd(batch, G, N).to(io), "D": rnd(dim),
            "dt_bias": 0.1 * rnd(dim)}
    res = []
    for guarded in (False, True):
        ar = Arena(guarded)
        t = {k: ar.inp(v) for k, v in vals.items()}
        st = ar.out((batch, dim, N), torch.float32)
        st.copy_(state0.to(DEV))
        out = ar.out((batch, dim), io)
        rc = _abi.lib().ssm_state_update_ex(p(st), p(t["x"]), p(t["dt"]), p(t["A"]), p(t["B"]),
                                            p(t["C"]), p(t["D"]), p(t["z"]), p(t["dt_bias"]), 1,
                                            p(out), batch, dim, N, G, IO_CODE[io], flags, 0)
        _abi.check(rc, "ssm_state_update_ex")
        ar.check_margins()
        res.append([out.clone(), st.clone()])
    same(res[1], res[0])
    assert ssm._abi.wait_timeouts() == 0
