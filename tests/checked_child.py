"""Child process of test_gpu_checked.py: runs a set of library calls with
whichever library OT_CHECKED selects and saves their outputs and the device
status of each group (the library loads once per process)."""

from __future__ import annotations

import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import torch  # noqa: E402

import unified_transformer_recommender_onetrans_b200 as ot  # noqa: E402
from gpu_common import make_model  # noqa: E402
from helpers import rand_inputs, rand_weights  # noqa: E402


def status(m) -> int:
    try:
        m.poll()
        return 0
    except ot.OtError as e:
        return e.code


def main(path: str) -> None:
    out, st = {}, {}
    # bf16 tcgen05: encode + score, the merged full forward, a paged cache
    shapes = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])
    w = rand_weights(3, 128, 256, 5, seed=501, dtype=torch.bfloat16)
    S, ns = rand_inputs(3, 4, 300, 5, 128, seed=502, dtype=torch.bfloat16)
    m = make_model(w, **shapes)
    S, ns = S.cuda(), ns.cuda()
    kv, s_tail = m.encode_user(S)
    out["bf16_s"], out["bf16_ns"] = s_tail, m.score_candidates(kv, ns)
    out["full_s"], out["full_ns"] = m.full_forward(S, ns)
    pool = m.new_page_pool(3 * m.kv_pages_per_user())
    pages = torch.arange(3 * m.kv_pages_per_user(), dtype=torch.int32).view(3, -1).cuda()
    out["paged_s"] = m.encode_user_paged(S, pool, pages)
    out["paged_ns"] = m.score_candidates_paged(pool, pages, ns)
    st["bf16"] = status(m)
    # fp32 on the CUDA-core kernels
    wf = rand_weights(2, 64, 128, 3, seed=503)
    Sf, nsf = rand_inputs(2, 3, 70, 3, 64, seed=504)
    mf = make_model(wf, layers=2, d=64, heads=2, ffn=128, n_ns=3, L0=70, q=[70, 20], dtype="f32")
    out["f32_s"], out["f32_ns"] = mf.full_forward(Sf.cuda(), nsf.cuda())
    st["f32"] = status(mf)
    torch.save({"out": {k: v.cpu() for k, v in out.items()}, "status": st}, path)


if __name__ == "__main__":
    main(sys.argv[1])
