"""GPU-side test fixtures: upload synthetic layers, quantize them with the CUDA kernel, and check
the codes against the oracle's on the way.  Imported by the `-m gpu` tests only."""
import numpy as np
import torch

import int8_expert_weight_b200 as jm
import oracle
import synth
from helpers import gap_inputs


def bf16_to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_to_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class Layer:
    """Inputs and weights of one workload: host copies for the oracle, device copies for the GPU.
    Weights are generated per expert, quantized on the GPU, and (if check_quant) compared bit for
    bit with the oracle's quantization of the same bf16 values."""

    def __init__(self, wl: synth.Workload, check_quant: bool = True, keep_host_q: bool = True):
        self.wl = wl
        inp = gap_inputs(wl)
        self.x_bits, self.wr, self.bias = inp["x"], inp["wr"], inp["bias"]
        self.redrawn = inp["redrawn"]
        self.x = bf16_to_dev(self.x_bits)
        self.wr_dev = torch.from_numpy(self.wr).cuda()
        self.bias_dev = None if self.bias is None else torch.from_numpy(self.bias).cuda()
        self.q, self.s, self.qh, self.sh = {}, {}, {}, {}
        self.quant_mismatch = {}
        for which in ("w1", "w3", "w2"):
            rows, cols = synth.weight_shape(wl, which)
            Q = torch.empty((wl.E, rows, cols), dtype=torch.int8, device="cuda")
            S = torch.empty((wl.E, rows), dtype=torch.float32, device="cuda")
            qh = np.empty((wl.E, rows, cols), dtype=np.int8) if keep_host_q else None
            sh = np.empty((wl.E, rows), dtype=np.float32) if keep_host_q else None
            bad = 0
            for e in range(wl.E):
                w = synth.gen_expert(wl, which, e)
                jm.jamba_moe_quantize(bf16_to_dev(w), out=(Q[e], S[e]))
                if check_quant or keep_host_q:
                    qo, so = oracle.quantize(w)
                    if check_quant:
                        bad += int(np.count_nonzero(Q[e].cpu().numpy() != qo))
                        bad += int(np.count_nonzero(S[e].cpu().numpy().view(np.uint32) != so.view(np.uint32)))
                    if keep_host_q:
                        qh[e], sh[e] = qo, so
            self.q[which], self.s[which] = Q, S
            self.qh[which], self.sh[which] = qh, sh
            self.quant_mismatch[which] = bad
        torch.cuda.synchronize()

    def forward(self, path=jm.PATH_AUTO, workspace=None):
        y, ids, w = jm.jamba_moe_forward(self.x, self.wr_dev, self.bias_dev, self.q["w1"], self.s["w1"],
                                         self.q["w3"], self.s["w3"], self.q["w2"], self.s["w2"],
                                         workspace=workspace, path=path)
        torch.cuda.synchronize()
        return dev_to_bf16_bits(y), ids.cpu().numpy(), w.cpu().numpy()

    def oracle_forward(self, tokens=None, want_hidden=False):
        return oracle.moe_forward(self.x_bits, self.wr, self.bias, self.qh["w1"], self.sh["w1"], self.qh["w3"],
                                  self.sh["w3"], self.qh["w2"], self.sh["w2"], tokens=tokens,
                                  want_hidden=want_hidden)
