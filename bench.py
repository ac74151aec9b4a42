#!/usr/bin/env python
"""Benchmark of the Hidden Decoding hot path on B200 (one JSON line on rank 0).

One step = one pass of every hot-path operation, each at its own workload
configuration's sizes, over synthetic inputs resident in HBM, in this order:
  x   hd_expand_embed, ids [4, 8192] -> X [4, 32768, 4096] from 4 fp32 tables
  c5  hd_decode_attn, CROSS_FULL and INTRA, 4 new stream queries per sequence
      against a 16384-token cache, batch 8 and batch 64
  c2  hd_attn_fwd + hd_attn_bwd, INTRA: B4 n4 L2048 (8192 expanded positions),
      16 query / 4 KV heads, head_dim 128
  c3  hd_attn_fwd + hd_attn_bwd, CROSS_WINDOW (W = 1024 tokens = 4096
      positions): B2 n4 L8192 (32768 positions), 32 / 8 heads
  c4  hd_attn_fwd, CROSS_FULL over 131072 positions, and final-stream-only
      queries (KV-mirror, 32768 rows) with their hd_attn_bwd: B1 n4 L32768,
      32 / 8 heads
value = unmasked attention TFLOP/s over the step (fwd 4*D, bwd 10*D FLOPs per
visible (query, key, head) pair, decode 4*D per pair); per_op carries every
operation's time, TFLOP/s or GB/s and roofline fraction.

--workload selects another measurement: step_intra_train (every row at the
intra-stream layer's sizes, a 10 ms step), intra_train, cross_window,
long_cross, long_cross_train (fwd/bwd of one configuration), cross_full_32k
(CROSS_FULL fwd+bwd over 32768 positions), decode8 /
decode64 / decode8_final (decode steps), expand, rope (RoPE of q and k at
131072 positions), lm_head and lm_head_train (final-stream LM-head
cross-entropy, and with its gradients). HBM-bound workloads report GB/s, the
rest TFLOP/s.

--impl reference times the float64 CPU oracle (the reference arm) on a bounded
sample of the same workload. Multi-GPU (torchrun): every rank runs its own
replica of the step (data parallel, no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

INTRA, CROSS_FULL, CROSS_WINDOW = 0, 1, 2
METRIC = "unmasked attention TFLOP/s & expanded tokens/s (fwd+bwd); decode µs/step, GB/s"

# Sizes of the five workload configurations the hot path is measured on (V and
# d size the expansion tables; T is the decode cache's prior tokens).
CFG = {
    # intra-stream training layer
    "c2": dict(B=4, L=2048, n=4, Hq=16, Hkv=4, D=128, W=1024, V=32000, d=2048, T=2048),
    # cross-stream sliding-window layer, window 1024 tokens = 4096 positions
    "c3": dict(B=2, L=8192, n=4, Hq=32, Hkv=8, D=128, W=1024, V=32000, d=4096, T=8192),
    # long-context full cross-stream layer (+ final-stream-only queries, KV-mirror)
    "c4": dict(B=1, L=32768, n=4, Hq=32, Hkv=8, D=128, W=1024, V=32000, d=4096, T=32768),
    # multi-stream decode step against a 16384-token cache, batch 8 and 64
    "c5b8": dict(B=8, L=1, n=4, Hq=32, Hkv=8, D=128, W=1024, V=32000, d=4096, T=16384),
    "c5b64": dict(B=64, L=1, n=4, Hq=32, Hkv=8, D=128, W=1024, V=32000, d=4096, T=16384),
    # embedding expansion: 4 fp32 tables of 32000 x 4096, 32768 tokens
    "x": dict(B=4, L=8192, n=4, Hq=32, Hkv=8, D=128, W=1024, V=32000, d=4096, T=1),
}
WL = CFG["c2"]


# ------------------------------------------------------------------ counting
def pairs(S, n, mode, W, final_only):
    """Visible (query, key) pairs of one (batch, head) problem (closed forms)."""
    L = S // n
    if final_only:
        if mode == INTRA:
            return L * (L + 1) // 2
        # row t at position t*n + n-1 sees min(p+1, n*W) keys
        tot = 0
        lim = n * W if mode == CROSS_WINDOW else None
        p = np.arange(L, dtype=np.int64) * n + (n - 1)
        vis = p + 1 if lim is None else np.minimum(p + 1, lim)
        tot = int(vis.sum())
        return tot
    if mode == INTRA:
        return n * L * (L + 1) // 2
    if mode == CROSS_FULL:
        return S * (S + 1) // 2
    w = min(n * W, S)
    return w * (w + 1) // 2 + (S - w) * w


def decode_pairs(n, T, mode):
    """Visible cache positions summed over the n stream queries of one (b, h)."""
    if mode == INTRA:
        return n * (T + 1)
    return sum(T * n + s + 1 for s in range(n))


def step_plan(wl):
    B, n, L, Hq, Hkv, D, W, T = (wl[k] for k in ("B", "n", "L", "Hq", "Hkv", "D", "W", "T"))
    S = n * L
    ops = []
    for name, mode, fin in (("intra", INTRA, 0), ("cross_full", CROSS_FULL, 0),
                            ("cross_window", CROSS_WINDOW, 0), ("final_only", CROSS_FULL, 1)):
        pr = pairs(S, n, mode, W, fin) * B * Hq
        ops.append(dict(name=f"fwd_{name}", kind="fwd", mode=mode, fin=fin, flops=4 * D * pr, pairs=pr))
        ops.append(dict(name=f"bwd_{name}", kind="bwd", mode=mode, fin=fin, flops=10 * D * pr, pairs=pr))
    for name, mode in (("cross_full", CROSS_FULL), ("intra", INTRA)):
        pr = decode_pairs(n, T, mode) * B * Hq
        kv_bytes = 2 * B * (T + 1) * n * Hkv * D * 2
        io = B * n * Hq * D * 2 * 2 + B * Hq * n * 4
        ops.append(dict(name=f"decode_{name}", kind="decode", mode=mode, fin=0, flops=4 * D * pr,
                        pairs=pr, bytes=kv_bytes + io))
    for name, mode in (("cross_full", CROSS_FULL), ("intra", INTRA)):
        # final stream alone: INTRA reads only that stream's T+1 rows
        rows = (T + 1) * (n if mode == CROSS_FULL else 1)
        pr = B * Hq * rows
        kv_bytes = 2 * B * rows * Hkv * D * 2
        io = B * Hq * D * 2 * 2 + B * Hq * 4
        ops.append(dict(name=f"decode_final_{name}", kind="decode_final", mode=mode, fin=1,
                        flops=4 * D * pr, pairs=pr, bytes=kv_bytes + io))
    ex_bytes = B * L * 4 + 2 * B * L * n * wl["d"] * 4
    ops.insert(0, dict(name="expand", kind="expand", flops=0, pairs=0, bytes=ex_bytes))
    # final-stream LM-head cross-entropy: one GEMM of the B*L final rows with the head
    ops.append(dict(name="lm_head_ce", kind="lm_head", flops=2 * B * L * wl["d"] * wl["V"], pairs=0))
    # its gradients: logits recomputed, dh = G W, dW = G^T h (three GEMMs of the same size)
    ops.append(dict(name="lm_head_ce_bwd", kind="lm_head_bwd", flops=3 * 2 * B * L * wl["d"] * wl["V"], pairs=0))
    # rotary embedding of q and k in place: every element read and written once
    ops.append(dict(name="rope", kind="rope", flops=0, pairs=0, bytes=2 * 2 * B * S * (Hq + Hkv) * D))
    return ops


LAUNCHES = {"expand": 1, "fwd": 1, "bwd": 3, "decode": 2, "decode_final": 2, "rope": 1, "lm_head": 2,
            "lm_head_bwd": 3}

# A workload is a list of parts: (label, sizes, operation names of step_plan).
# The default "step" is one pass of every hot-path row at the configurations'
# own sizes; the others measure one configuration (or one supplementary kernel).
WORKLOADS = {
    # the expansion and the decode steps first, then the training layers from
    # the shortest to the long-context one (whose ~230 ms hold the GPU at its
    # power cap, so whatever follows it starts at a lowered clock)
    "step": [("x", CFG["x"], ["expand"]),
             ("c5b8", CFG["c5b8"], ["decode_cross_full", "decode_intra"]),
             ("c5b64", CFG["c5b64"], ["decode_cross_full", "decode_intra"]),
             ("c2", CFG["c2"], ["fwd_intra", "bwd_intra"]),
             ("c3", CFG["c3"], ["fwd_cross_window", "bwd_cross_window"]),
             ("c4", CFG["c4"], ["fwd_cross_full", "fwd_final_only", "bwd_final_only"])],
    # every row at the intra-stream layer's sizes in one short step (decode
    # against a 2048-token cache)
    "step_intra_train": [("", CFG["c2"], ["expand", "fwd_intra", "bwd_intra", "fwd_cross_full", "bwd_cross_full",
                                          "fwd_cross_window", "bwd_cross_window", "fwd_final_only",
                                          "bwd_final_only", "decode_cross_full", "decode_intra"])],
    "intra_train": [("", CFG["c2"], ["fwd_intra", "bwd_intra"])],
    "cross_window": [("", CFG["c3"], ["fwd_cross_window", "bwd_cross_window"])],
    "long_cross": [("", CFG["c4"], ["fwd_cross_full", "fwd_final_only"])],
    "long_cross_train": [("", CFG["c4"], ["fwd_final_only", "bwd_final_only"])],
    # a mid-size full-causal layer (the long-problem grid orders, ~1 GB on the
    # device): the case the detailed profiles of the long kernels are taken on
    "cross_full_32k": [("", dict(CFG["c4"], L=8192, T=8192), ["fwd_cross_full", "bwd_cross_full"])],
    "decode8": [("", CFG["c5b8"], ["decode_cross_full", "decode_intra"])],
    "decode64": [("", CFG["c5b64"], ["decode_cross_full", "decode_intra"])],
    "decode8_final": [("", CFG["c5b8"], ["decode_final_cross_full", "decode_final_intra"])],
    "expand": [("", CFG["x"], ["expand"])],
    "lm_head": [("", dict(CFG["c3"], T=1), ["lm_head_ce"])],
    "lm_head_train": [("", dict(CFG["c3"], T=1), ["lm_head_ce", "lm_head_ce_bwd"])],
    "rope": [("", dict(CFG["c4"], T=1), ["rope"])],
}


def plan_for(name):
    """[(label, sizes, ops)] of a workload; op names get the part's label as prefix."""
    parts = []
    for label, wl, names in WORKLOADS[name]:
        by_name = {o["name"]: o for o in step_plan(dict(wl))}
        ops = []
        for nm in names:
            o = dict(by_name[nm])
            o["op"] = nm
            o["name"] = f"{label}.{nm}" if label else nm
            ops.append(o)
        parts.append((label, dict(wl), ops))
    return parts


# --------------------------------------------------------------- GPU state
class Part:
    """Device buffers of one configuration plus the calls of its operations.

    Only the buffers its operations use are allocated.
    """

    def __init__(self, wl, ops, dev):
        import structured_causal_attention_b200 as hd
        from structured_causal_attention_b200 import synthetic as syn

        self.hd, self.wl, self.dev = hd, wl, dev
        B, n, L, Hq, Hkv, D, V, d, T = (wl[k] for k in ("B", "n", "L", "Hq", "Hkv", "D", "V", "d", "T"))
        S = n * L
        kinds = {o["kind"] for o in ops}
        attn = kinds & {"fwd", "bwd"}
        fin = any(o.get("fin") for o in ops if o["kind"] in ("fwd", "bwd"))
        full = any(not o.get("fin") for o in ops if o["kind"] in ("fwd", "bwd"))
        bwd_fin = any(o.get("fin") for o in ops if o["kind"] == "bwd")
        bwd_full = any(not o.get("fin") for o in ops if o["kind"] == "bwd")
        # host copies (pinned) of every per-step input, for the end-to-end leg
        self.h = {}
        if "expand" in kinds:
            self.h["ids"] = syn.token_ids(B, L, V, seed=9)
        if attn:
            a = syn.attention_inputs(B, L, n, Hq, Hkv, D, seed=2, with_grad=bwd_full)
            self.h.update({"k": a["k"], "v": a["v"]})
            if full:
                self.h["q"] = a["q"]
                if bwd_full:
                    self.h["do"] = a["do"]
            if fin:
                self.h["qf"] = syn.normal_bf16((B, L, Hq, D), 12)
                if bwd_fin:
                    self.h["dof"] = syn.normal_bf16((B, L, Hq, D), 13)
        if "decode" in kinds:
            self.h["dq_new"] = syn.normal_bf16((B, n, Hq, D), 14)
        if "decode_final" in kinds:
            self.h["dq_fin"] = syn.normal_bf16((B, 1, Hq, D), 18)
        if kinds & {"lm_head", "lm_head_bwd"}:
            li = syn.lm_head_inputs(B, L, n, d, V, seed=19)
            self.h["x_hid"] = li["x"]
            self.h["labels"] = li["labels"]
        if "rope" in kinds and not attn:
            self.h["q"] = syn.normal_bf16((B, S, Hq, D), 16)
            self.h["k"] = syn.normal_bf16((B, S, Hkv, D), 17)
        for k_ in list(self.h):
            self.h[k_] = self.h[k_].pin_memory()
        self.d = {k_: v_.to(dev) for k_, v_ in self.h.items()}
        # a second set of device inputs: the end-to-end leg copies step i+1's
        # inputs into one set while step i computes on the other
        self.d_alt = {k_: torch.empty_like(v_) for k_, v_ in self.d.items()}
        g = torch.Generator(device=dev)
        g.manual_seed(15)
        # model state kept resident: embedding tables and the KV cache
        if "expand" in kinds:
            self.tables = torch.empty((n, V, d), dtype=torch.float32, device=dev).normal_(0, 0.02, generator=g)
            self.x = torch.empty((B, S, d), dtype=torch.float32, device=dev)
        if kinds & {"decode", "decode_final"}:
            self.kc = torch.empty((B, (T + 1) * n, Hkv, D), dtype=torch.bfloat16, device=dev).normal_(generator=g)
            self.vc = torch.empty_like(self.kc).normal_(generator=g)
            self.seqlen = torch.full((B,), T + 1, dtype=torch.int32, device=dev)
        if "decode" in kinds:
            self.ws_dec_n = hd.hd_decode_workspace_bytes(B, n, T + 1, Hq, Hkv, D)
            self.ws_dec = torch.empty(self.ws_dec_n, dtype=torch.uint8, device=dev)
            self.dec_o = {m: torch.empty_like(self.d["dq_new"]) for m in ("cross_full", "intra")}
            self.dec_l = {m: torch.empty((B, Hq, n), dtype=torch.float32, device=dev)
                          for m in ("cross_full", "intra")}
        if kinds & {"lm_head", "lm_head_bwd"}:
            self.w_head = torch.empty((V, d), dtype=torch.bfloat16, device=dev).normal_(0, 3.0 / math.sqrt(d), generator=g)
            self.loss = torch.empty((B, L), dtype=torch.float32, device=dev)
            self.loss_lse = torch.empty((B, L), dtype=torch.float32, device=dev)
            self.ws_lm_n = hd.hd_lm_head_ce_workspace_bytes(B, L, V)
            self.ws_lm = torch.empty(self.ws_lm_n, dtype=torch.uint8, device=dev)
        if "lm_head_bwd" in kinds:
            self.dh = torch.empty((B, L, d), dtype=torch.bfloat16, device=dev)
            self.dw_head = torch.empty((V, d), dtype=torch.float32, device=dev)
            self.ws_lmb_n = hd.hd_lm_head_ce_bwd_workspace_bytes(B, L, V)
            self.ws_lmb = torch.empty(self.ws_lmb_n, dtype=torch.uint8, device=dev)
        if "decode_final" in kinds:
            self.ws_fin_n = hd.hd_decode_final_workspace_bytes(B, n, T + 1, Hq, Hkv, D)
            self.ws_fin = torch.empty(self.ws_fin_n, dtype=torch.uint8, device=dev)
            self.fin_o = {m: torch.empty_like(self.d["dq_fin"]) for m in ("cross_full", "intra")}
            self.fin_l = {m: torch.empty((B, Hq, 1), dtype=torch.float32, device=dev)
                          for m in ("cross_full", "intra")}
        self.o, self.lse = {}, {}
        for o in ops:
            if o["kind"] == "fwd":
                key = o["op"].split("_", 1)[1]
                rows = L if o["fin"] else S
                self.o[key] = torch.empty((B, rows, Hq, D), dtype=torch.bfloat16, device=dev)
                self.lse[key] = torch.empty((B, Hq, rows), dtype=torch.float32, device=dev)
        if "bwd" in kinds:
            if bwd_full:
                self.dq = torch.empty_like(self.d["q"])
            if bwd_fin:
                self.dqf = torch.empty_like(self.d["qf"])
            self.dk = torch.empty_like(self.d["k"])
            self.dv = torch.empty_like(self.d["v"])
            self.ws_bwd_n = hd.hd_attn_bwd_workspace_bytes(B, L, n, Hq, Hkv, D, 0 if bwd_full else 1)
            self.ws_bwd = torch.empty(self.ws_bwd_n, dtype=torch.uint8, device=dev)
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in self.h.values())
        # the part's result read back to the host: decode outputs, else the first forward's LSE
        self.result = []
        if "decode" in kinds:
            self.result += list(self.dec_o.values())
        elif "decode_final" in kinds:
            self.result += list(self.fin_o.values())
        elif self.lse:
            self.result.append(next(iter(self.lse.values())))
        elif "expand" in kinds:
            self.result.append(self.x[:, :1])
        elif "rope" in kinds:
            self.result.append("k")  # a slice of the step's own input set (see results())
        elif "lm_head" in kinds:
            self.result.append(self.loss)
        self.host_res = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in self.results(self.d)]
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.results(self.d))

    def results(self, d):
        """The part's result tensors for input set d (read back to the host)."""
        return [d[t][:, :1] if isinstance(t, str) else t for t in self.result]

    def call(self, op, stream, d=None):
        hd, wl = self.hd, self.wl
        d = self.d if d is None else d
        B, n, L, Hq, Hkv, D, W, T = (wl[k] for k in ("B", "n", "L", "Hq", "Hkv", "D", "W", "T"))
        sc = 1.0 / math.sqrt(D)
        s = stream.cuda_stream
        name = op["op"]
        if op["kind"] == "expand":
            hd.hd_expand_embed(d["ids"], self.tables, self.x, B, L, n, wl["V"], wl["d"], 4, s)
        elif op["kind"] == "lm_head":
            hd.hd_lm_head_ce(d["x_hid"], self.w_head, d["labels"], self.loss, self.loss_lse, B, L, n,
                             wl["d"], wl["V"], self.ws_lm, self.ws_lm_n, s)
        elif op["kind"] == "lm_head_bwd":
            hd.hd_lm_head_ce_bwd(d["x_hid"], self.w_head, d["labels"], self.loss_lse, 1.0, self.dh,
                                 self.dw_head, B, L, n, wl["d"], wl["V"], self.ws_lmb, self.ws_lmb_n, s)
        elif op["kind"] == "rope":
            hd.hd_rope_expanded(d["q"], d["k"], None, B, L, n, Hq, Hkv, D, 0, 10000.0, s)
        elif op["kind"] in ("fwd", "bwd"):
            key = name.split("_", 1)[1]
            fin = op["fin"]
            q = d["qf"] if fin else d["q"]
            if op["kind"] == "fwd":
                hd.hd_attn_fwd(q, d["k"], d["v"], self.o[key], self.lse[key], B, L, n, Hq, Hkv, D,
                               op["mode"], W, fin, sc, s)
            else:
                do = d["dof"] if fin else d["do"]
                hd.hd_attn_bwd(q, d["k"], d["v"], self.o[key], self.lse[key], do,
                               self.dqf if fin else self.dq, self.dk, self.dv, B, L, n, Hq, Hkv, D,
                               op["mode"], W, fin, sc, self.ws_bwd, self.ws_bwd_n, s)
        elif op["kind"] == "decode_final":
            key = name.split("_", 2)[2]
            hd.hd_decode_attn_final(d["dq_fin"], self.kc, self.vc, self.seqlen, self.fin_o[key],
                                    self.fin_l[key], B, n, T + 1, Hq, Hkv, D, op["mode"], W, sc,
                                    self.ws_fin, self.ws_fin_n, s)
        else:
            key = name.split("_", 1)[1]
            hd.hd_decode_attn(d["dq_new"], self.kc, self.vc, self.seqlen, self.dec_o[key],
                              self.dec_l[key], B, n, T + 1, Hq, Hkv, D, op["mode"], W, sc,
                              self.ws_dec, self.ws_dec_n, s)

    def h2d(self, d):
        """Copy the part's inputs from pinned host memory into input set d (current stream)."""
        for k_, v_ in self.h.items():
            d[k_].copy_(v_, non_blocking=True)

    def d2h(self, d):
        """Copy the part's result back into pinned host memory (current stream)."""
        for h_, t_ in zip(self.host_res, self.results(d)):
            h_.copy_(t_, non_blocking=True)


class Step:
    """The parts of a workload and its operations in step order: (part index, op)."""

    def __init__(self, parts, dev):
        self.parts = [Part(wl, ops, dev) for _, wl, ops in parts]
        self.ops = [(i, o) for i, (_, _, ops) in enumerate(parts) for o in ops]
        self.flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.h2d_bytes = sum(p.h2d_bytes for p in self.parts)
        self.d2h_bytes = sum(p.d2h_bytes for p in self.parts)

    def input_sets(self):
        """The two device input sets, each a list with one dict per part."""
        return [[p.d for p in self.parts], [p.d_alt for p in self.parts]]

    def call(self, k, stream, dset=None):
        i, op = self.ops[k]
        self.parts[i].call(op, stream, None if dset is None else dset[i])

    def h2d(self, dset):
        for p, d in zip(self.parts, dset):
            p.h2d(d)

    def d2h(self, dset):
        for p, d in zip(self.parts, dset):
            p.d2h(d)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        self.index = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- CPU oracle leg
_ORACLE_INPUTS = {}


def _oracle_inputs(label, wl):
    """float64 copies of batch 0 of a configuration's synthetic inputs (cached)."""
    if label not in _ORACLE_INPUTS:
        from structured_causal_attention_b200 import synthetic as syn

        B, n, L, Hq, Hkv, D = (wl[k] for k in ("B", "n", "L", "Hq", "Hkv", "D"))
        a = syn.attention_inputs(1, L, n, Hq, Hkv, D, seed=2)
        t = {k: a[k].to(torch.float64).numpy() for k in ("q", "k", "v")}
        t["qf"] = syn.normal_bf16((1, L, Hq, D), 12).to(torch.float64).numpy()
        _ORACLE_INPUTS[label] = t
    return _ORACLE_INPUTS[label]


def oracle_sample(budget_s, parts, seed=0):
    """Time the float64 oracle on a bounded sample of the step's attention work.

    Returns (unmasked FLOPs done, seconds, description). Each draw takes 32
    random query rows of one random head of every forward operation of the
    step, at that operation's own sizes (batch 0), and is credited 4*D FLOPs
    per visible pair.
    """
    import oracle

    rng = np.random.default_rng(seed)
    cases = [(label, wl, o) for label, wl, ops in parts for o in ops if o["kind"] == "fwd"]
    for label, wl, _ in cases:
        _oracle_inputs(label, wl)
    flops, t0, nrows = 0, time.perf_counter(), 0
    while time.perf_counter() - t0 < budget_s:
        for label, wl, o in cases:
            n, L, Hq, D, W = (wl[k] for k in ("n", "L", "Hq", "D", "W"))
            a64 = _oracle_inputs(label, wl)
            fin, mode = o["fin"], o["mode"]
            h = int(rng.integers(Hq))
            rows = rng.choice(L if fin else n * L, 32, replace=False)
            q = a64["qf"] if fin else a64["q"]
            oracle.attn_fwd_rows(q, a64["k"], a64["v"], n, mode, W, bool(fin), 1.0 / math.sqrt(D), 0, h, rows)
            pos = rows * n + (n - 1) if fin else rows
            if mode == INTRA:
                vis = (pos // n + 1) if not fin else (rows + 1)
            elif mode == CROSS_FULL:
                vis = pos + 1
            else:
                vis = np.minimum(pos + 1, n * W)
            flops += int(4 * D * vis.sum())
            nrows += len(rows)
    dt = time.perf_counter() - t0
    names = ", ".join(o["name"] for _, _, o in cases)
    return flops, dt, f"{nrows} query rows (32 per draw) of the forward operations {names}, batch 0, " \
                      f"random heads, float64 oracle"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        th = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(th) if th else os.cpu_count()
    except Exception:
        return os.cpu_count()


# ------------------------------------------------------------------ ranks
def reduce_max(values, device):
    """Max over ranks of a list of floats (the timing rule for N > 1)."""
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_value(flops_per_step, world, ms_per_step):
    """Whole-job TFLOP/s: every rank runs its own replica of the step."""
    return flops_per_step * max(world, 1) / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------- main
DESCRIPTIONS = {
    "step": "every hot-path row at the configurations' own sizes: c2 INTRA fwd+bwd B4 n4 L2048 Hq16 Hkv4 D128; "
            "c3 CROSS_WINDOW fwd+bwd B2 n4 L8192 W1024 tokens Hq32 Hkv8; c4 CROSS_FULL fwd (131072 queries) and "
            "final-stream-only fwd+bwd (32768 queries) B1 n4 L32768 Hq32 Hkv8; c5 decode CROSS_FULL + INTRA, "
            "16384-token cache, B8 and B64; x expansion B4 L8192 n4 V32000 d4096 fp32",
    "step_intra_train": "every row at the intra_train sizes: B4 n4 L2048 (8192 expanded positions), Hq16 Hkv4 "
                        "D128; expand (V32000 d2048 fp32 tables) + fwd/bwd INTRA, CROSS_FULL, CROSS_WINDOW(W=1024 "
                        "tokens), final-stream-only + decode (cache 2048 tokens, CROSS_FULL and INTRA)",
    "intra_train": "INTRA fwd+bwd, B4 n4 L2048 (8192 expanded), Hq16 Hkv4 D128",
    "cross_window": "CROSS_WINDOW fwd+bwd, B2 n4 L8192 (32768 expanded), W=1024 tokens, Hq32 Hkv8 D128",
    "long_cross": "CROSS_FULL fwd (131072 queries) + final-stream-only fwd (32768 queries), B1 n4 L32768, "
                  "Hq32 Hkv8 D128",
    "long_cross_train": "final-stream-only fwd+bwd (32768 queries, 131072 keys), B1 n4 L32768, Hq32 Hkv8 D128",
    "cross_full_32k": "CROSS_FULL fwd+bwd, B1 n4 L8192 (32768 expanded), Hq32 Hkv8 D128",
    "decode8": "decode step CROSS_FULL + INTRA, B8 n4, 16384 prior tokens (65540 cache rows), Hq32 Hkv8 D128",
    "decode64": "decode step CROSS_FULL + INTRA, B64 n4, 16384 prior tokens (65540 cache rows), Hq32 Hkv8 D128",
    "expand": "expansion B4 L8192 n4, V32000, d4096 fp32 tables",
    "decode8_final": "final-stream-only decode (one query per sequence) CROSS_FULL + INTRA, B8 n4, "
                     "16384 prior tokens (65540 cache rows), Hq32 Hkv8 D128",
    "lm_head": "final-stream readout + fused LM-head cross-entropy, x [2,32768,4096] bf16 (16384 final-stream "
               "rows), head [32000,4096] bf16",
    "lm_head_train": "final-stream LM-head cross-entropy and its gradients (dh, dW), x [2,32768,4096] bf16 "
                     "(16384 final-stream rows), head [32000,4096] bf16",
    "rope": "RoPE in place at physical positions, q [1,131072,32,128] + k [1,131072,8,128] bf16, base 10000",
}

# DRAM bytes per launch of the dominant kernel from the last ncu capture of
# the same build (dram__bytes_read.sum + dram__bytes_write.sum); a workload
# whose dominant kernel changed after its capture has no entry (null).
NCU_TRAFFIC = {
    ("step", "c4.fwd_cross_full"): 4.24e9,            # attn_fwd_tc_kernel (--workload long_cross)
    ("long_cross", "fwd_cross_full"): 4.24e9,         # attn_fwd_tc_kernel
    ("long_cross_train", "bwd_final_only"): 6.58e9,   # attn_bwd_tc_kernel
    ("cross_window", "bwd_cross_window"): 18.74e9,    # attn_bwd_tc_kernel
    ("step_intra_train", "bwd_cross_full"): 4.13e9,   # attn_bwd_tc_kernel
    ("cross_full_32k", "bwd_cross_full"): 17.24e9,    # attn_bwd_tc_kernel
    ("lm_head", "lm_head_ce"): 2.280e9,               # lm_head_ce_kernel
    ("rope", "rope"): 2.628e9,                        # rope_kernel
}

KERNELS = {"fwd": "hd_attn_fwd (attn_fwd_tc_kernel)",
           "bwd": "hd_attn_bwd (bwd_pre + attn_bwd_tc_kernel + bwd_dq)",
           "decode": "hd_decode_attn (decode_split + decode_combine)",
           "expand": "hd_expand_embed (expand_kernel)",
           "decode_final": "hd_decode_attn_final (decode_split + decode_combine)",
           "rope": "hd_rope_expanded (rope_kernel)",
           "lm_head": "hd_lm_head_ce (lm_head_ce_kernel + lm_head_combine)",
           "lm_head_bwd": "hd_lm_head_ce_bwd (gradient pass + two gemm_tc_kernel)"}
TENSOR_KINDS = ("fwd", "bwd", "lm_head", "lm_head_bwd")
HBM_KINDS = ("decode", "decode_final", "expand", "rope")


def roofline_of(op, ms, peaks):
    """Roofline record of one operation from its mean CUDA-event time.

    Tensor-core operations are compared with the measured burst bf16 GEMM
    rate (frac) and, beside it, with the sustained one (frac_of_sustained);
    HBM-bound ones with the measured copy bandwidth.
    """
    burst = peaks.get("bf16_tflops", 1590.0)
    sustained = peaks.get("bf16_tflops_sustained", 1400.0)
    hbm = peaks.get("hbm_gbs", 6650.0)
    src = "MEASURED_PEAKS.json" if peaks else "fallback"
    if op["kind"] in TENSOR_KINDS:
        ach = op["flops"] / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": round(ach, 1), "peak": burst, "unit": "TFLOP/s",
                "frac": round(ach / burst, 4), "peak_source": f"{src} bf16_tflops (burst)",
                "frac_of_sustained": round(ach / sustained, 4)}
    ach = op["bytes"] / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
            "peak_source": f"{src} hbm_gbs"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="step", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    parts = plan_for(args.workload)
    ops = [o for _, _, pops in parts for o in pops]
    total_flops = sum(o["flops"] for o in ops)
    total_bytes = sum(o.get("bytes", 0) for o in ops)
    hbm_only = total_flops == 0 or all(o["kind"] in HBM_KINDS for o in ops)
    attn_parts = [wl for _, wl, pops in parts if any(o["kind"] in ("fwd", "bwd") for o in pops)]
    tokens = sum(wl["B"] * wl["n"] * wl["L"] for wl in attn_parts)
    big = max((wl for _, wl, _ in parts), key=lambda w: w["B"] * w["n"] * w["L"])
    config = {"workload": DESCRIPTIONS[args.workload],
              "global_batch": big["B"] * max(world, 1), "seq_len": big["n"] * big["L"],
              "parallelism": f"replicas{max(world, 1)}",
              "l2": "256 MB buffer written between timed steps (outside the per-step events); "
                    "per-step working set larger than L2"}

    if args.impl == "reference":
        if rank != 0:
            return
        budget = 2.0
        vals = []
        for i in range(args.warmup + args.steps):
            fl, dt, desc = oracle_sample(budget, parts, seed=i)
            if i >= args.warmup:
                vals.append((fl, dt))
        fl = sum(v[0] for v in vals)
        dt = sum(v[1] for v in vals)
        val = fl / dt / 1e12
        out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
               "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
               "data": "synthetic", "config": config,
               "cpu_baseline": {"kind": "oracle", "value": val, "unit": "TFLOP/s", "cores": blas_threads(),
                                "sample": f"each step: ~{budget:.0f} s of " + desc},
               "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(out))
        return

    # ---------------- our CUDA library
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from structured_causal_attention_b200.build import build

    if rank == 0 or world == 1:
        build()
    if world > 1:
        dist.barrier()
    import structured_causal_attention_b200 as hd

    hd.lib()
    st = Step(parts, dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    def one_step(evs=None, dset=None):
        for i in range(len(st.ops)):
            if evs is not None:
                evs[i][0].record(stream)
            st.call(i, stream, dset)
            if evs is not None:
                evs[i][1].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one_step()
    torch.cuda.synchronize()
    if hd.hd_device_status() != hd.HD_OK:
        raise RuntimeError("device status set during warm-up")

    # ---------------- device-timed steps (inputs resident in HBM)
    op_ms = [[] for _ in ops]
    step_ms = []
    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for _ in range(args.steps):
            with torch.cuda.stream(stream):
                st.flush.zero_()
                evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in ops]
                one_step(evs)
            stream.synchronize()
            for i, (a, b) in enumerate(evs):
                op_ms[i].append(a.elapsed_time(b))
            step_ms.append(evs[0][0].elapsed_time(evs[-1][1]))
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    clocks = clk.summary()
    total_ms = sum(step_ms)

    # ---------------- end to end: pinned host inputs -> device -> result back to host.
    # Every step's inputs are copied inside the timed region, on a copy stream
    # that runs one step ahead (step i+1's copy overlaps step i's kernels, as a
    # training input pipeline does); each step's result is read back after it.
    n_e2e = max(3, args.steps // 2)
    copy_stream = torch.cuda.Stream(device=dev)
    sets = st.input_sets()
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e_start.record(stream)
    copy_stream.wait_event(e_start)
    with torch.cuda.stream(copy_stream):
        st.h2d(sets[0])
        copied[0].record(copy_stream)
    for i in range(n_e2e):
        b = i % 2
        if i + 1 < n_e2e:
            with torch.cuda.stream(copy_stream):
                if i >= 1:
                    copy_stream.wait_event(consumed[1 - b])  # step i-1 is done with that set
                st.h2d(sets[1 - b])
                copied[1 - b].record(copy_stream)
        with torch.cuda.stream(stream):
            stream.wait_event(copied[b])
            one_step(dset=sets[b])
            consumed[b].record(stream)
            st.d2h(sets[b])
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_step = e_start.elapsed_time(e_end) / n_e2e
    if hd.hd_device_status() != hd.HD_OK:
        raise RuntimeError("device status set during timing")

    if world > 1:
        total_ms, e2e_step = reduce_max([total_ms, e2e_step], dev)
    ms_step = total_ms / args.steps

    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    per_op = {}
    wl_of = {o["name"]: wl for _, wl, pops in parts for o in pops}
    for op, ms in zip(ops, op_ms):
        m = sum(ms) / len(ms)
        rec = {"ms": round(m, 4)}
        if op["kind"] in TENSOR_KINDS or op.get("bytes"):
            r = roofline_of(op, m, peaks)
            rec["tflops" if r["unit"] == "TFLOP/s" else "gbs"] = r["achieved"]
            rec["frac"] = r["frac"]
            if "frac_of_sustained" in r:
                rec["frac_of_sustained"] = r["frac_of_sustained"]
        if op["kind"] in ("fwd", "bwd"):
            wl = wl_of[op["name"]]
            rows = wl["B"] * wl["L"] * (1 if op["fin"] else wl["n"])
            rec["query_rows_per_s" if op["fin"] else "expanded_tokens_per_s"] = round(rows / (m * 1e-3), 1)
        if op["kind"] in ("decode", "decode_final"):
            rec["us"] = round(1e3 * m, 2)
        per_op[op["name"]] = rec
    dom = max(ops, key=lambda o: per_op[o["name"]]["ms"])
    roof = roofline_of(dom, per_op[dom["name"]]["ms"], peaks)
    roof = {"kernel": f"{KERNELS[dom['kind']]}, op {dom['name']}", **roof,
            "traffic": NCU_TRAFFIC.get((args.workload, dom["name"]))}
    if hbm_only:
        value = total_bytes * max(world, 1) / (ms_step * 1e-3) / 1e9
        e2e_val = total_bytes * max(world, 1) / (e2e_step * 1e-3) / 1e9
        unit = "GB/s"
    else:
        value = whole_job_value(total_flops, world, ms_step)
        e2e_val = whole_job_value(total_flops, world, e2e_step)
        unit = "TFLOP/s"
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": max(world, 1),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config,
        "e2e": {"value": round(e2e_val, 2), "unit": unit,
                "h2d_bytes_per_step": st.h2d_bytes, "d2h_bytes_per_step": st.d2h_bytes,
                "ms_per_step": round(e2e_step, 4), "steps": n_e2e,
                "pipeline": "step i+1's host-to-device copy overlaps step i's kernels; inputs larger "
                            "than L2, no flush between steps"},
        "gpu_launches": args.steps * sum(LAUNCHES[o["kind"]] for o in ops),
        "roofline": roof,
        "per_op": per_op,
        "clocks": clocks,
    }
    if tokens and not hbm_only:
        out["expanded_tokens_per_s"] = round(tokens * max(world, 1) / (ms_step * 1e-3), 1)
    dec = next((per_op[o["name"]] for o in ops if o["kind"] == "decode" and o["mode"] == CROSS_FULL), None)
    if dec:
        out["decode_us_per_step"] = dec["us"]
        out["decode_gbs"] = dec.get("gbs")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        fl, dt, desc = oracle_sample(10.0, parts)
        out["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                               "kind": "oracle", "sample": f"{dt:.1f} s: " + desc}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


if __name__ == "__main__":
    main()
