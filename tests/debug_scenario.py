"""One seeded run of the library, printed as a JSON line of output digests.

tests/test_gpu_debug_build.py runs this script in child processes, once with the release
library and once with the debug build (ZO_LIB=debug, device bounds checks), and compares
the digests: the checks must not change a bit, and no check may fire on valid input.

    python tests/debug_scenario.py model          # probe steps (fp32, bf16), generation
    python tests/debug_scenario.py attention DIR  # the tensor-core attention op; the output
                                                  # goes to DIR/attention.npy as float32
"""
import dataclasses
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from zeroth_order_fine_b200 import workload as wl  # noqa: E402
from zeroth_order_fine_b200 import zo  # noqa: E402
from gpu_util import dev_tokens, gpu_handle  # noqa: E402

# rows of 1 to 300 tokens (ragged last tiles, several 128-query tiles per row); the last row
# is shorter than one tile, so its only tile is the last one after the longest-first sort
ATTN_LENS = [1, 129, 300, 256, 77]
ATTN_H, ATTN_HKV = 4, 2


def digest(*arrays) -> str:
    h = hashlib.sha256()
    for a in arrays:
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                a = a.view(torch.int16)
            a = a.numpy()
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def steps(w, shape, n_steps, nu):
    batch = wl.make_batch(w)
    toks = dev_tokens(batch)
    _, h = gpu_handle(w, shape=shape, nu=nu)
    out = []
    for t in range(n_steps):
        h.zo_probe_plan(t, w.eps)
        Lp, Lm, lp = h.zo_score(toks, batch.seq_lens, batch.target_lens, want_logprob=True)
        c = h.zo_step(w.lr)
        out.append(digest(Lp, Lm, lp, np.float64(c)))
    out.append(hashlib.sha256(h.zo_save_state()).hexdigest())
    h.close()
    return out


def generation(w, shape):
    batch = wl.make_batch(w, batch=2)
    toks = dev_tokens(batch)
    _, h = gpu_handle(w, shape=shape, batch=2, max_new=4)
    h.zo_probe_plan(0, w.eps)
    Lp, Lm, gt, gl = h.zo_generate(toks, batch.seq_lens, 4)
    c = h.zo_step(w.lr)
    res = digest(Lp, Lm, gt, gl, np.float64(c))
    h.close()
    return res


def model_part():
    w = wl.WORKLOADS["tiny"]
    bf16 = wl.shrink_shape(w.shape, dtype=wl.DTYPE_BF16)
    w_bf = dataclasses.replace(w, shape=bf16)
    return {
        "fp32_steps": steps(w, None, 3, 2),
        "bf16_steps": steps(w_bf, bf16, 3, 2),
        "bf16_generation": generation(w_bf, bf16),
    }


def attention_part(out_dir):
    g = torch.Generator().manual_seed(31)
    T = sum(ATTN_LENS)
    qkv = torch.randn(T, (ATTN_H + 2 * ATTN_HKV) * 128, generator=g).to(torch.bfloat16).cuda()
    out = torch.full((T, ATTN_H * 128), 7.0, dtype=torch.bfloat16, device="cuda")
    zo.zo_op_attention(qkv, ATTN_LENS, ATTN_H, ATTN_HKV, 128, impl=zo.IMPL_TENSOR_CORES, out=out)
    torch.cuda.synchronize()
    np.save(os.path.join(out_dir, "attention.npy"), out.float().cpu().numpy())
    return {"attention": digest(out)}


def main():
    part = sys.argv[1]
    res = model_part() if part == "model" else attention_part(sys.argv[2])
    torch.cuda.synchronize()
    res["debug_build"] = int(zo.lib().zo_debug_build())
    res["debug_word"] = int(zo.lib().zo_debug_word(1))
    print(json.dumps(res))


if __name__ == "__main__":
    main()
