"""Steps a mixed tensor list through whichever library ADAMW4_LIBRARY names
and prints a hash of the weights and state (run as a child process by
test_gpu_checked.py, so each build loads in its own process)."""
import hashlib
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def main():
    import torch
    import bit_quantized_optimizer_b200 as B
    import workloads
    BF, Q = B.ADAMW4_T_BF16_PARAM, B.ADAMW4_T_QUANT_STATE
    specs = [dict(numel=128 * 300 + 5, tensor_id=1, flags=0, weight_decay=0.1),
             dict(numel=4096, tensor_id=2, flags=workloads.T_LM_HEAD, weight_decay=0.0),
             dict(numel=3000, tensor_id=3, flags=0, weight_decay=0.1),
             dict(numel=5000, tensor_id=4, flags=workloads.T_NORM, weight_decay=0.0),
             dict(numel=128 * 90 + 7, tensor_id=5, flags=BF, weight_decay=0.1),
             dict(numel=1280, tensor_id=6, flags=Q, weight_decay=0.1, elem_offset=128 * 40)]
    out = {}
    for vcode in range(5):
        params, grads = [], []
        for i, s in enumerate(specs):
            w = torch.from_numpy((np.random.default_rng(i).standard_normal(s["numel"]) * 0.02)
                                 .astype(np.float32)).cuda()
            params.append(w.to(torch.bfloat16) if s["flags"] & BF else w)
            grads.append(torch.zeros(s["numel"], dtype=torch.bfloat16, device="cuda"))
        opt = B.AdamW4(params, grads, specs, vcode=vcode, seed=5, total_steps=3)
        h = hashlib.sha256()
        for t in range(3):
            for i, (g, s) in enumerate(zip(grads, specs)):
                hg = workloads.bf16_bits((np.random.default_rng(100 * t + i).standard_normal(
                    s["numel"]) * 1e-3).astype(np.float32))
                g.view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
            opt.step()
            opt.sync()                       # raises on ADAMW4_ECHECK / ADAMW4_ETIMEOUT
        for p in params:
            h.update(p.view(torch.int16).cpu().numpy().tobytes() if p.dtype == torch.bfloat16
                     else p.cpu().numpy().tobytes())
        h.update(opt.state_dict_blob())
        opt.close()
        out[vcode] = h.hexdigest()
    print(json.dumps({"lib": B.LIB_PATH, "hashes": out}))


if __name__ == "__main__":
    main()
