"""The debug build: bounds-checked kernels with the release build's results.

``libdmuon_b200_debug.so`` (``build.py --debug``, also made by
``__graft_entry__.build()``) checks every global access of its kernels against
the extent of the buffer it belongs to; an access outside is skipped and the
device status word records DMUON_ERR_BOUNDS.  Each library is loaded in a child
process (DMUON_LIBRARY) that runs the same calls on ragged shapes of every path
(tensor-core pair and one-CTA kernels, FFMA kernels, the clustered thin-matrix
chain, elementwise and clip kernels, the fused update, overlapped chunks) and
saves its outputs.  The debug run must record no bounds error and give the
release run's bits; its self-test must show that the checks are live.
"""
import os
import subprocess
import sys

import pytest
import torch

from tests.gpu_util import bits

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "newton_schulz_grad_b200")
RELEASE = os.path.join(PKG, "libdmuon_b200.so")
DEBUG = os.path.join(PKG, "libdmuon_b200_debug.so")

BATTERY = r'''
import os, sys, torch
import newton_schulz_grad_b200 as nsg
import workloads
res = {"info": nsg.dmuon_build_info(), "status": {}}
dev = "cuda"
gen = torch.Generator().manual_seed(3)

def done(tag):
    res["status"][tag] = nsg.dmuon_stream_status()

for r, c in [(1, 37), (37, 1), (100, 37), (257, 129), (130, 136), (300, 520), (520, 300),
             (1408, 2048), (64, 4100), (33, 1000), (384, 1100)]:
    for dt in (torch.bfloat16, torch.float32):
        x = torch.randn(r, c, generator=gen).to(dt).to(dev)
        out = torch.empty_like(x)
        nsg.dmuon_ns(x, out, steps=5)
        done(f"ns {r}x{c} {dt}")
        res[f"ns {r}x{c} {dt}"] = out.cpu()

os.environ["DMUON_WS_CAP_MB"] = "64"   # several chunks, overlapped
w = workloads.get("small_layer_bf16")
ps, gs, bs = workloads.make_all(w, dev)
nsg.dmuon_step(ps, gs, bs, wd=0.1)
done("step small")
res["step small"] = [t.cpu() for t in ps + bs]
ps, gs, bs = workloads.make_all(w, dev)
nsg.dmuon_step(ps, gs, bs, max_norm=0.5)
done("clipped step small")
res["clipped step small"] = [t.cpu() for t in ps + bs]
del os.environ["DMUON_WS_CAP_MB"]

w = workloads.get("moe_skewed_bf16")
sk = workloads.skewed_indices(w)
mats = [workloads.make_matrix(w, i, dev, sk) for i in (0, 2, 192, 193, 240)]
ps, gs, bs = [m[0] for m in mats], [m[1] for m in mats], [m[2] for m in mats]
nsg.dmuon_step(ps, gs, bs)
done("step moe")
res["step moe"] = [t.cpu() for t in ps + bs]

w = workloads.get("single_256x512_f32")
ps, gs, bs = workloads.make_all(w, dev)
nsg.dmuon_step(ps, gs, bs, ns_steps=0, wd=0.5)
nsg.dmuon_step(ps, gs, bs)
done("step f32")
res["step f32"] = [t.cpu() for t in ps + bs]

grads = [torch.randn(r, c, generator=gen).to(torch.bfloat16).to(dev) for r, c in [(100, 37), (257, 129), (5, 4099)]]
grads.append(torch.randn(1, 64 * 37 + 3, generator=gen).to(dev)[0, 3:].view(64, 37))
nsg.dmuon_clip_grad_norm(grads, 1.0, float("inf"))
done("clip")
res["clip"] = [g.cpu() for g in grads]

x = torch.randn(300, 520, generator=gen).to(torch.bfloat16).to(dev)
out = torch.empty_like(x)
word = torch.zeros(1, dtype=torch.int32, device=dev)
nsg.dmuon_ns_noalloc(x, out, steps=5, status=word)
done("noalloc")
res["status"]["noalloc word"] = int(word.item())
res["noalloc"] = out.cpu()

g = torch.randn(130, 77, generator=gen).to(torch.bfloat16).to(dev)
buf = torch.randn(130, 77, generator=gen).to(torch.bfloat16).to(dev)
x0 = torch.empty_like(g)
nsg.dmuon_momentum(buf, g, x0, 0.9, True)
p = torch.randn(130, 77, generator=gen).to(torch.bfloat16).to(dev)
nsg.dmuon_update(p, x0, 0.02, 0.1)
done("stages")
res["stages"] = [buf.cpu(), x0.cpu(), p.cpu()]

nsg.dmuon_selftest_bounds()
res["selftest"] = nsg.dmuon_stream_status()
res["after selftest"] = nsg.dmuon_stream_status()
torch.save(res, sys.argv[1])
'''


def run_battery(lib, out):
    env = dict(os.environ, DMUON_LIBRARY=lib)
    subprocess.run([sys.executable, "-c", BATTERY, str(out)], check=True, cwd=ROOT, env=env, timeout=900)
    return torch.load(out)


def flat(v):
    return v if isinstance(v, list) else [v]


def test_debug_build_is_bounds_clean_and_bit_identical(tmp_path):
    assert os.path.exists(DEBUG), "build it with `python newton_schulz_grad_b200/build.py --debug`"
    rel = run_battery(RELEASE, tmp_path / "release.pt")
    dbg = run_battery(DEBUG, tmp_path / "debug.pt")
    assert "release" in rel["info"] and "debug bounds checks" in dbg["info"]
    # no access fell outside its buffer, in either build
    assert all(v == 0 for v in dbg["status"].values()), {k: v for k, v in dbg["status"].items() if v}
    assert all(v == 0 for v in rel["status"].values())
    # the checks are live in the debug build only, and the status clears
    assert dbg["selftest"] == 6 and dbg["after selftest"] == 0
    assert rel["selftest"] == 0
    keys = [k for k in rel if k not in ("info", "status", "selftest", "after selftest")]
    assert len(keys) > 20
    for k in keys:
        for a, b in zip(flat(rel[k]), flat(dbg[k])):
            assert torch.equal(torch.from_numpy(bits(a)), torch.from_numpy(bits(b))), k
