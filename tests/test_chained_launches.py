"""Back-to-back library calls on one stream, with no host synchronisation between them.

Every kernel of the library is launched with programmatic dependent launch: it may be
scheduled while the previous kernel on the stream is still running, and waits
(griddepcontrol.wait) before its first global access. These cases chain calls whose
buffers depend on each other in both directions (read after write: a kernel reads
what the previous one wrote; write after read: a kernel overwrites what the previous
one reads) and compare every result with the same calls run one at a time with a
synchronisation after each.
"""
import pytest
import torch

import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs

pytestmark = pytest.mark.gpu


def run_chain(x, g, w, sync):
    dev = x.device
    step = (lambda: torch.cuda.synchronize()) if sync else (lambda: None)
    out = {}
    qf = q.quantize_fwd(x, 4, mask_mode=q.MASK_BITS); step()
    out["codes"], out["mask"], out["scales"] = qf["codes"].clone(), qf["mask"], qf["scales"].clone()
    step()
    out["gin"] = q.trust_bwd(g, qf["mask"]); step()                       # reads the mask just written
    ox, ow = q.quantize_operands(x, w); step()
    cx = ox["codes"].view(torch.int8).reshape(x.shape)
    cw = ow["codes"].view(torch.int8).reshape(w.shape)
    out["y"] = q.w4a4_linear(cx, ox["scales"], cw, ow["scales"]); step()   # reads both operands
    # write after read: the transpose overwrites the weight that the quantizer just
    # launched is reading (its source is a copy made before)
    scratch = w.clone(); step()
    wq = q.quantize_fwd(w, 4, rms_group=w.shape[1], code_mode=q.CODES_GEMM_OPERAND, mask_mode=None); step()
    n_out, k_in = w.shape
    wt_dst = w.view(k_in, n_out)                                        # same storage as w
    q.transpose_bf16(scratch, out=wt_dst); step()                       # w's storage now holds w^T
    out["wq_codes"] = wq["codes"]
    out["w_after"] = w.clone()
    gy = inputs.upstream_grad(x.shape[0], n_out, seed=3).to(dev)
    out["gx"] = q.trust_bwd_linear(gy, wt_dst, qf["mask"]); step()       # reads w^T and the mask
    torch.cuda.synchronize()
    return out


def test_chain_matches_synchronised_calls(cuda_device):
    dev = torch.device("cuda:0")
    x0 = inputs.activation_input(rows=2048).to(dev)
    g0 = inputs.grad_input(rows=2048).to(dev)
    w0 = inputs.weight_up(rows=768).to(dev)
    ref = run_chain(x0.clone(), g0.clone(), w0.clone(), sync=True)
    for _ in range(3):
        got = run_chain(x0.clone(), g0.clone(), w0.clone(), sync=False)
        q.device_status()
        for k in ref:
            a, b = got[k], ref[k]
            if a.dtype == torch.bfloat16:
                a, b = a.view(torch.int16), b.view(torch.int16)
            assert torch.equal(a, b), k
