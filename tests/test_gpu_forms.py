"""Both forms of the assignment kernel -- one CTA per 128-point tile, and
two-SM CTA pairs on 256-point tiles -- against the oracle.  The form is fixed
per process (KM_ASSIGN_FORM), so each runs in a child process that writes its
outputs to a file; the comparisons happen here."""

import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import oracle
from tests.parity import JTOL, check_assignment

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys, torch
    import means_clustering_flashassign_b200 as km
    from synth import WORKLOADS, make_problem
    out = {}
    g = torch.Generator().manual_seed(11)
    Xi = torch.randint(-3, 4, (5000, 64), generator=g).to(torch.bfloat16)
    Ci = torch.randint(-3, 4, (700, 64), generator=g).to(torch.bfloat16)
    Ci[400:500] = Ci[0:100]
    Xi[:64] = Ci[:64]
    out["int"] = [t.cpu() for t in km.assign(Xi.cuda(), Ci.cuda())[:2]]
    for N, D, K, B in [(3001, 128, 300, 1), (20000, 128, 1000, 1), (1000, 256, 129, 1), (2000, 64, 256, 3)]:
        wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K, B=B)
        X, C, _ = make_problem(wl, seed=N + K, device="cuda")
        idx, md, obj = km.assign(X.contiguous(), C.contiguous())
        out[(N, D, K, B)] = (X.cpu(), C.cpu(), idx.cpu(), md.cpu(), obj.cpu())
    torch.cuda.synchronize()
    torch.save(out, sys.argv[1])
""")


@pytest.mark.parametrize("form", ["single", "pair"])
def test_assign_forms_match_oracle(form, tmp_path):
    path = str(tmp_path / f"{form}.pt")
    env = dict(os.environ, KM_ASSIGN_FORM=form, PYTHONPATH=ROOT)
    subprocess.run([sys.executable, "-c", CHILD, path], env=env, cwd=ROOT, check=True, timeout=600)
    out = torch.load(path)
    # integer data: every score exact, so idx and mindist match bit for bit
    g = torch.Generator().manual_seed(11)
    Xi = torch.randint(-3, 4, (5000, 64), generator=g).to(torch.bfloat16)
    Ci = torch.randint(-3, 4, (700, 64), generator=g).to(torch.bfloat16)
    Ci[400:500] = Ci[0:100]
    Xi[:64] = Ci[:64]
    io, d1, _ = oracle.assign(Xi, Ci)
    assert np.array_equal(out["int"][0].numpy(), io)
    assert np.array_equal(out["int"][1].double().numpy(), d1)
    for key, val in out.items():
        if key == "int":
            continue
        X, C, idx, md, obj = val
        B = key[3]
        for b in range(B):
            Xb, Cb = (X[b], C[b]) if B > 1 else (X, C)
            ib, mb = (idx[b], md[b]) if B > 1 else (idx, md)
            r = check_assignment(Xb, Cb, ib, mb, "bf16")
            J = r["d1"].sum()
            ob = obj[b] if B > 1 else obj.reshape(-1)[0]
            assert abs(ob.item() - J) <= JTOL * J + r["jfloor"], (key, b)
