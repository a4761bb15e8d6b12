"""One small, fixed MoBA case on cuda:0, for capturing a kernel under a profiler.

    python -m block_sparse_long_11_b200.profile_case --op forward --tokens 65536 \
        --chunk-tokens 16384
    python -m block_sparse_long_11_b200.profile_case --op gate --tokens 262144
    python -m block_sparse_long_11_b200.profile_case --op decode --tokens 262144 --seqs 2

Shape: one sequence, 32 query heads over 8 KV heads, head dim 128, block 4096,
top-k 12 (the Llama-8B-1M setting of the MoBA write-up, "大語言模型評估"
section), seeded synthetic bf16 inputs.  The op runs ``--reps`` times, so a
capture can skip the first (cold) launch of the kernel it wants.  ``decode``
runs one decode step of ``--seqs`` sequences whose caches hold ``--tokens``
tokens (block means filled first).
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import block_sparse_long_11_b200 as mb  # noqa: E402
import synth  # noqa: E402


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--op", choices=["forward", "gate", "decode"], default="forward")
    ap.add_argument("--seqs", type=int, default=2)
    ap.add_argument("--tokens", type=int, default=65536)
    ap.add_argument("--chunk-tokens", type=int, default=None)
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--seed", type=int, default=5)
    a = ap.parse_args(argv)
    B, topk = 4096, 12
    if a.op == "decode":
        x = synth.make_decode(a.seqs, a.tokens, 32, 8, 128, seed=a.seed, device="cuda")
        sl = torch.full((a.seqs,), a.tokens - 7, dtype=torch.int32, device="cuda")
        kbar = mb.moba_decode_init(x["k_cache"], sl, B)
        for _ in range(a.reps):
            res = mb.moba_decode(x["q"], x["k_cache"], x["v_cache"], sl, kbar, B, topk)[0]
        mb.moba_check()
        torch.cuda.synchronize()
        print(f"ok decode seqs={a.seqs} context={a.tokens - 7} "
              f"result_sum={float(res.float().sum()):.6g} "
              f"peak_mem={torch.cuda.max_memory_allocated() / 2**30:.2f} GiB")
        return
    _, x = synth.make_custom([a.tokens], 32, 8, 128, B, topk, seed=a.seed, device="cuda")
    for _ in range(a.reps):
        if a.op == "forward":
            res = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], B, topk,
                                  chunk_tokens=a.chunk_tokens)[0]
        else:
            res = mb.moba_gate(x["q"], x["k"], x["cu_seqlens"], B, topk)
    mb.moba_check()
    torch.cuda.synchronize()
    print(f"ok {a.op} tokens={a.tokens} result_sum={float(res.float().sum()):.6g} "
          f"peak_mem={torch.cuda.max_memory_allocated() / 2**30:.2f} GiB")


if __name__ == "__main__":
    main()
