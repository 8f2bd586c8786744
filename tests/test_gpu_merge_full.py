"""The full adapter-merge workload: 36 layers x 7 targets of a 2560-hidden
model (q 2560->4096, k/v 2560->1024, o 4096->2560, gate/up 2560->9728,
down 9728->2560), r = 32, alpha = 64, all 252 matrices in one batched call,
ten perturb + restore + merge refreshes.

Checked: every matrix's rows sampled per 128-row tile against the oracle
within the merge bound, and within one bf16 ULP on every element whose
fp32 accumulation does not cancel; the pristine copies bit-identical after the ten
cycles (SHA-256); each refresh's merged state equal to a second merge of
the same adapter from pristine, bit for bit."""
import hashlib

import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import dev, f64
from tolerance import merge_tol_check

pytestmark = pytest.mark.gpu


def _sha(t):
    return hashlib.sha256(t.contiguous().view(torch.int16).cpu().numpy().tobytes()).hexdigest()


def test_full_merge_workload(gpu):
    r, alpha = WL.MERGE_R, WL.MERGE_ALPHA
    shapes = WL.merge_shapes()
    assert len(shapes) == 252
    L = gpu
    pristine, hosts, rows_of, W_rows = [], [], [], []
    for i, s in enumerate(shapes):
        m = WL.make_merge_inputs(s["d_out"], s["d_in"], r, seed=1000 + i)
        pristine.append(dev(m["W"]))
        rows = WL.sample_rows(s["d_out"], seed=i, per_tile=1)
        rows_of.append(rows)
        W_rows.append(m["W"][rows].clone())     # keep only the sampled rows on the host
        hosts.append(dict(A=m["A"], B=m["B"]))
    h0 = [_sha(p) for p in pristine]
    W_inf = [torch.empty_like(p) for p in pristine]

    for cycle in range(10):
        A_c, B_c = [], []
        for i, m in enumerate(hosts):
            a, b = WL.perturb_adapter(m["A"], m["B"], cycle, seed=5000 + i)
            A_c.append(dev(a))
            B_c.append(dev(b))
        for i in range(len(shapes)):
            L.lora_restore(pristine[i], W_inf[i])
        L.lora_merge_batched(list(zip(pristine, A_c, B_c, W_inf)), r, alpha)
        assert L.lora_get_device_status() == 0
        if cycle in (0, 9):
            again = [torch.empty_like(p) for p in pristine]
            L.lora_merge_batched(list(zip(pristine, A_c, B_c, again)), r, alpha)
            for x, y in zip(W_inf, again):
                assert torch.equal(x, y)
        if cycle == 9:
            for i in range(len(shapes)):
                rows = rows_of[i]
                Wr = f64(W_rows[i])
                rd = rows.cuda()
                Af, Bf = f64(A_c[i].cpu()), f64(B_c[i][rd].cpu())
                exact = O.lora_merge(Wr, Af, Bf, alpha)
                ok, info = merge_tol_check(f64(W_inf[i][rd].cpu()), exact, Wr, Af, Bf, alpha / r)
                assert ok, (i, shapes[i], info)
                # one ULP wherever the fp32 accumulation cannot cancel
                assert info["max_ulps_noncancel"] <= 1.0 and info["frac_noncancel"] > 0.9, (i, shapes[i], info)
    assert [_sha(p) for p in pristine] == h0
