"""CPU oracle for the packed-cache path — TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct restatement (numpy, fp64 unless a step's
precision is part of the definition) of what the method computes:

  codebooks.py  Lloyd-Max N(0,1) codebooks and the NF4 table
  rope.py       the RoPE block decomposition the method is built on
  blockgtq.py   energy score, greedy bit allocation, TQ-MSE-style quantizer,
                the packed tile layout and fused decode attention
  nqkv.py       NQKV-style per-block NF4 quantizer, layout and attention

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
leg may import this package. The CUDA library (libkvq) shares no code with it
and never calls it; nothing here imports the CUDA path.

Sources: "RoPE-aware bit allocation for KV cache quantization" (Liang, Zhang,
Jia; arXiv 2606.24033), abstract; "NQKV: A KV Cache Quantization Scheme Based
on Normal Distribution Characteristics" (Cai et al.; arXiv 2505.16210) as read
by its pith.science review: reading, referee report (major comment 1),
assumptions, Figs. 4-7; QLoRA (Dettmers et al.), cited there as reference
[20], for the NF4 construction. Where the pages leave a step open, each
function states the reading it takes.

Parity status: every function here is pinned by tests/test_oracle_pins.py
against closed forms, textbook constants, brute force or invariants; none is
"parity unpinned" except the absolute NF4 table values, which are pinned to
the QLoRA paper's published table rather than to the pages.
"""
