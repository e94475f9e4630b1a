"""F4 against bf16 K/V: how far decode attention over the F4 cache lands
from the same attention over the unquantised bf16 K/V.

The mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and hybrid
paged attention for Qwen3.5-Next long-context serving" (Known limitations)
records that F4-vs-BF16 equivalence at long context was never measured; the
ignis docs "context-and-speculation" name bf16 the format every correctness
oracle runs against. Both sides here are the fp64 oracle on the same inputs:
rotary on q and the new key, the F4 write of the context and the new token,
then exact attention over the F4 cache (oracle.paged_attention) and over the
bf16 rows (oracle.dense_attention).

    python oracle/f4_deviation.py [--tokens N] [workload ...]

Test infrastructure like the rest of oracle/: nothing in the product path
imports it.
"""
from __future__ import annotations

import argparse
import dataclasses
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
import workloads  # noqa: E402


def sample(w: workloads.Workload, n_tok: int) -> workloads.Workload:
    """The workload's recipe on one sequence of n_tok context tokens (the
    step's position and YaRN settings unchanged)."""
    L = min(n_tok, w.seq_lens[0])
    return dataclasses.replace(w, name=w.name + f"_{L}", n_layers=1, seq_lens=(L,),
                               num_pages=-(-L // w.block_size),
                               first_position=w.first_position + w.seq_lens[0] - L)


def deviation(w: workloads.Workload) -> dict:
    x = workloads.host_layer(w)
    spec = workloads.yarn_spec(w)
    q = oracle.rope_apply_bf16(x["q"], x["positions"], spec)
    k_new = oracle.rope_apply_bf16(x["k_new"], x["positions"], spec)
    cache = oracle.empty_cache(w.num_pages, w.kv_heads, w.block_size, w.head_dim)
    oracle.kv_write_f4(x["k_cache"], x["v_cache"], x["cache_slots"], cache, w.kv_heads, w.head_dim, w.block_size)
    oracle.kv_write_f4(k_new, x["v_new"], x["step_slots"], cache, w.kv_heads, w.head_dim, w.block_size)
    o4, l4 = oracle.paged_attention(q, cache, x["page_table"], [0], x["seq_lens"], w.q_heads, w.kv_heads,
                                    w.head_dim, w.block_size)
    k = np.concatenate([x["k_cache"], k_new])
    v = np.concatenate([x["v_cache"], x["v_new"]])
    ob, lb = oracle.dense_attention(q[0], k, v)
    d = o4[0] - ob
    return {"workload": w.name, "tokens": w.seq_lens[0], "max_abs_out": float(np.abs(d).max()),
            "rms_out": float(np.sqrt((d ** 2).mean())), "rel_out": float(np.linalg.norm(d) / np.linalg.norm(ob)),
            "max_abs_lse2": float(np.abs(l4[0] - lb).max()), "max_abs_ref_out": float(np.abs(ob).max())}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=65536)
    ap.add_argument("names", nargs="*", default=[w.name for w in workloads.ALL])
    a = ap.parse_args()
    print("| workload | context tokens | max abs(out) err | rms err | rel err (L2) | max abs lse2 err | max abs(out) |")
    print("|---|---|---|---|---|---|---|")
    for name in a.names:
        r = deviation(sample(workloads.BY_NAME[name], a.tokens))
        print(f"| {name} | {r['tokens']:,} | {r['max_abs_out']:.2e} | {r['rms_out']:.2e} | {r['rel_out']:.2e} | "
              f"{r['max_abs_lse2']:.2e} | {r['max_abs_ref_out']:.3f} |", flush=True)


if __name__ == "__main__":
    main()
