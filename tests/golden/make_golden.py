"""Writes ffn_reduced_w0.json: oracle outputs on a reduced tiny-FFN case.

The pages print no worked numerical example for SparseLoRA, so the only stored
expected values are these regression values, computed by the oracle alone
(this script imports nothing but the oracle and the seeded input module).
Run from the repository root:  python -m tests.golden.make_golden
"""
import json
import os

import numpy as np

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def compute():
    tok = synth.Tokens(batch=2, seq=24, ctx_len=np.array([18, 13], np.int32))
    case = synth.ffn_case(tok, d=32, d_ff=56, r_svd=4, r_lora=4, sparsity=0.5, workload=0, layer=9)
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=1.0)
    lay["Lg"], lay["Ug"] = O.svd_prepare(case.Wg.W, 4)
    lay["Lu"], lay["Uu"] = O.svd_prepare(case.Wu.W, 4)
    res = O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, 0.5)
    return dict(
        idx=[int(i) for i in res["idx"]],
        scores=[float(v) for v in res["scores"]],
        out_sum=[float(v) for v in res["out"].sum(axis=0)],
        dX_sum=[float(v) for v in res["dX"].sum(axis=0)],
        grad_norms=[float(np.linalg.norm(res[k])) for k in ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")],
    )


if __name__ == "__main__":
    with open(os.path.join(HERE, "ffn_reduced_w0.json"), "w") as f:
        json.dump(compute(), f, indent=1)
