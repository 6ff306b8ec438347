"""Named workloads (sizes and schedule parameters only).

The five attention-forward shapes the source pages are about (Llama-3 class
heads at 512 .. 1M tokens), each with the RoPE schedule it exercises.  Inputs
are synthetic: Q, K, V ~ N(0, 1), seed 0 (see inputs.py).
"""

from dataclasses import dataclass

PLAIN, PI, NTK, DYN_NTK, NTK_PARTS, YARN = range(6)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int
    dtype: str            # "f32" | "bf16"
    scheme: int
    base: float
    L_train: int
    L_target: int         # for DYN_NTK: the current sequence length l
    alpha: float = 1.0
    beta: float = 32.0
    window: int = 0
    n_sink: int = 0
    kv_block: int = 0     # ring block size in keys (0: one block)
    ring: bool = False    # run the multi-launch ring schedule (rcx_ring_attn_fwd)
    sample_rows: int = 0  # 0: compare every row with the oracle


WORKLOADS = {
    "pr1_fp32_512": Workload("pr1_fp32_512", 1, 1, 1, 64, 512, "f32", PI, 1e4, 256, 512,
                             kv_block=64, ring=True),
    "llama3_8b_8k": Workload("llama3_8b_8k", 1, 32, 8, 128, 8192, "bf16", NTK, 5e5, 8192, 32768,
                             kv_block=128),
    "llama3_70b_32k_yarn": Workload("llama3_70b_32k_yarn", 1, 64, 8, 128, 32768, "bf16", YARN, 1e4, 4096, 32768,
                                    alpha=1.0, beta=32.0, sample_rows=4096),
    "llama3_8b_128k_window": Workload("llama3_8b_128k_window", 1, 32, 8, 128, 131072, "bf16", DYN_NTK, 5e5, 8192,
                                      131072, window=4096, n_sink=4, sample_rows=4096),
    "llama3_70b_1m_ring": Workload("llama3_70b_1m_ring", 1, 64, 8, 128, 1 << 20, "bf16", NTK, 5e5, 8192, 1 << 20,
                                   kv_block=65536, ring=True, sample_rows=4096),
    # Three ring blocks of the 1M workload's shape (65,536 keys, same heads and
    # schedule): every launch form of the 1M ring (direct bf16 output, first,
    # middle and last partial) at 196,608 tokens, small enough to profile.
    "llama3_70b_192k_ring": Workload("llama3_70b_192k_ring", 1, 64, 8, 128, 3 * 65536, "bf16", NTK, 5e5, 8192,
                                     1 << 20, kv_block=65536, ring=True, sample_rows=4096),
    "llama3_8b_128k_ring": Workload("llama3_8b_128k_ring", 1, 32, 8, 128, 131072, "bf16", NTK, 5e5, 8192, 131072,
                                    kv_block=32768, ring=True, sample_rows=4096),
}

ORDER = ["pr1_fp32_512", "llama3_8b_8k", "llama3_70b_32k_yarn", "llama3_8b_128k_window", "llama3_8b_128k_ring",
         "llama3_70b_1m_ring"]
