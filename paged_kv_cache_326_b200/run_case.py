"""Run decode steps (write + paged attention) of one workload R times.

    python -m paged_kv_cache_326_b200.run_case [--workload NAME] [--num-seqs S] [--reps R]
                                               [--path fused|calls]

For profilers: it makes no timing claims.  Workloads: ``opt13b_batch64``
(optionally cut to the first S texts, pool sized 1.5x what they need),
``tiny``, ``skewed`` (bf16, blocks of 16), ``llama2_70b_gqa`` (64 query heads
on 8 key/value heads; always the two-call path, the one-launch step being
multi-head only), ``opt13b_batch64_fp8`` (the batch-64 step over 8-bit
caches, two calls), ``llama2_70b_gqa_fp8`` (the grouped-query step over
8-bit caches, two calls), ``opt13b_prefill`` (the prompt phase: S prompts of 2,048
tokens, 40 heads of 128; ``--prefill-kernel`` 0 automatic, 1 mma.sync, 2
tcgen05), ``shared_prefix`` (32 prompts x 8 samples built by the block
manager, through pa_paged_attn_decode_shared over the split tables).
``--gqa-kernel`` picks the grouped-query kernel (0 automatic, 1 CUDA cores, 2
tensor cores), ``--fp8-kernel`` the 8-bit one (same values).
``opt13b_prefill_reuse``: the prompt phase of the same prompts with their
first half already stored (pa_prefill_with_prefix; the first repetition
stores the whole prompts).
"""
from __future__ import annotations

import argparse

import torch

import paged_kv_cache_326_b200 as P
from paged_kv_cache_326_b200 import workloads as W


def make(name: str, num_seqs: int, device):
    if name == "tiny":
        return W.tiny(device=device)
    if name == "skewed":
        return W.skewed(device=device)
    if name == "opt13b_batch64_fp8":
        return W.opt13b_batch64_fp8(device=device)
    if name == "llama2_70b_gqa_fp8":
        return W.llama2_70b_gqa_fp8(device=device, num_seqs=num_seqs if num_seqs > 0 else 64)
    if name == "llama2_70b_gqa":
        return W.llama2_70b_gqa(device=device, num_seqs=num_seqs if num_seqs > 0 else 64)
    if name == "opt13b_batch64":
        if num_seqs <= 0 or num_seqs >= 64:
            return W.opt13b_batch64(device=device)
        lens = W.opt13b_batch64_lens()[:num_seqs]
        need = sum(W.blocks_needed(L, 16) for L in lens)
        return W.make_decode(f"opt13b_first{num_seqs}", lens, num_heads=40, head_dim=128,
                             block_size=16, num_blocks=(3 * need + 1) // 2, dtype=torch.float16,
                             seed=2, device=device, max_blocks_per_seq=128)
    raise SystemExit(f"unknown workload {name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="opt13b_batch64")
    ap.add_argument("--num-seqs", type=int, default=0)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--path", choices=["fused", "calls"], default="fused")
    ap.add_argument("--gqa-kernel", type=int, choices=[0, 1, 2], default=0)
    ap.add_argument("--prefill-kernel", type=int, choices=[0, 1, 2], default=0)
    ap.add_argument("--fp8-kernel", type=int, choices=[0, 1, 2], default=0)
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    P.pa_set_option(P.PA_OPT_FP8_KERNEL, args.fp8_kernel)
    if args.workload == "opt13b_prefill_reuse":
        w = W.opt13b_prefill(device=dev, num_prompts=args.num_seqs if args.num_seqs > 0 else 16)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        out = torch.empty_like(w.q)
        P.pa_prefill(out, w.q, w.k, w.v, w.cu_seqlens, w.max_seqlen, w.scale, w.k_cache,
                     w.v_cache, w.slot_mapping, status=status)
        L = w.lens[0]
        c = L // 2
        rows = torch.cat([torch.arange(int(w.cu_seqlens[s]) + c, int(w.cu_seqlens[s + 1]),
                                       device=dev) for s in range(len(w.lens))])
        qn, kn, vn = w.q[rows].contiguous(), w.k[rows].contiguous(), w.v[rows].contiguous()
        sn = w.slot_mapping[rows].contiguous()
        cun = torch.arange(0, (len(w.lens) + 1) * (L - c), L - c, dtype=torch.int32, device=dev)
        cached = torch.full((len(w.lens),), c, dtype=torch.int32, device=dev)
        outn = torch.empty_like(qn)
        for _ in range(args.reps):
            P.pa_prefill_with_prefix(outn, qn, kn, vn, cun, L - c, w.scale, w.k_cache, w.v_cache,
                                     w.block_tables, cached, sn, status=status)
        torch.cuda.synchronize()
        if status.item() != 0:
            raise SystemExit(f"device status {status.item()}: {P.pa_status_string(status.item())}")
        print(f"{len(w.lens)} prompts, {c} tokens stored, {L - c} new each, status ok")
        return
    if args.workload == "opt13b_prefill":
        P.pa_set_option(P.PA_OPT_PREFILL_KERNEL, args.prefill_kernel)
        w = W.opt13b_prefill(device=dev, num_prompts=args.num_seqs if args.num_seqs > 0 else 16)
        out = torch.empty_like(w.q)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        for _ in range(args.reps):
            P.pa_prefill(out, w.q, w.k, w.v, w.cu_seqlens, w.max_seqlen, w.scale, w.k_cache,
                         w.v_cache, w.slot_mapping, status=status)
        torch.cuda.synchronize()
        if status.item() != 0:
            raise SystemExit(f"device status {status.item()}: {P.pa_status_string(status.item())}")
        print(f"{len(w.lens)} prompts of {w.lens[0]} tokens, status ok")
        return
    if args.workload == "shared_prefix":
        bm = P.BlockManager(8192, 16)

        class Adapter:
            add_seq = staticmethod(bm.add_seq)
            fork = staticmethod(bm.fork)
            append_slot = staticmethod(bm.append_slot)
            export = staticmethod(lambda ids, m: tuple(t.numpy() for t in bm.export(ids, m)))

        w = W.shared_prefix(Adapter, num_blocks=8192, seed=4, device=dev)
        gs = w.meta["samples"]
        pt, pl, tt, tl = [t.to(dev) for t in P.split_shared_prefix(
            w.block_tables.cpu(), w.context_lens.cpu(), w.block_size, gs)]
        out = torch.empty_like(w.q)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        for _ in range(args.reps):
            P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=status)
            P.pa_paged_attn_decode_shared(out, w.q, w.k_cache, w.v_cache, pt, pl, tt, tl,
                                          w.scale, gs, status=status)
        torch.cuda.synchronize()
        if status.item() != 0:
            raise SystemExit(f"device status {status.item()}: {P.pa_status_string(status.item())}")
        print(f"shared_prefix: {w.num_seqs} texts in groups of {gs}, status ok")
        return
    w = make(args.workload, args.num_seqs, dev)
    gqa = w.k_cache.shape[1] != w.num_heads
    fp8 = w.k_cache.dtype == torch.uint8
    P.pa_set_option(P.PA_OPT_GQA_KERNEL, args.gqa_kernel)
    out = torch.empty_like(w.q)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(args.reps):
        if fp8:
            ks, vs = w.meta["k_scale"], w.meta["v_scale"]
            P.pa_kv_cache_write_fp8(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, ks, vs,
                                    status=status)
            P.pa_paged_attn_decode_fp8(out, w.q, w.k_cache, w.v_cache, w.block_tables,
                                       w.context_lens, w.scale, ks, vs, status=status)
        elif gqa:
            P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=status)
            P.pa_paged_attn_decode_gqa(out, w.q, w.k_cache, w.v_cache, w.block_tables,
                                       w.context_lens, w.scale, status=status)
        elif args.path == "fused":
            P.pa_decode_step(out, w.q, w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping,
                             w.block_tables, w.context_lens, w.scale, status=status)
        else:
            P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=status)
            P.pa_paged_attn_decode(out, w.q, w.k_cache, w.v_cache, w.block_tables,
                                   w.context_lens, w.scale, status=status)
    torch.cuda.synchronize()
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()}: {P.pa_status_string(status.item())}")
    kv = (sum(w.context_lens.tolist()) * 2 * w.k_cache.shape[1] * w.head_dim *
          w.k_cache.element_size())
    print(f"{w.name}: {w.num_seqs} texts, KV bytes per step {kv}, status ok")


if __name__ == "__main__":
    main()
