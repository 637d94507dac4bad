"""Named synthetic workloads (shapes only; inputs come from ``inputs.py``).

Shapes are those of the Llama-3.1 linear layers the ExLlamaV3 pages discuss
(8B: hidden 4096, intermediate 14336, 8 KV heads of 128; 70B: hidden 8192,
intermediate 28672, 8 KV heads; vocabulary 128256).  Each entry is
(name, m, k_in, n_out, K, outliers).
"""

# One linear layer 4096 x 4096 at K = 4, m = 1.
PR1 = [("pr1_4096x4096", 1, 4096, 4096, 4, False)]

# Llama-3.1-8B decode GEMV set: m = 1, K in {2,3,4,6,8}, four layer shapes.
LLAMA8B_SHAPES = [("q_o", 4096, 4096), ("k_v", 4096, 1024), ("gate_up", 4096, 14336),
                  ("down", 14336, 4096)]
LLAMA8B_DECODE = [("8b_%s_K%d" % (nm, K), 1, k, n, K, False)
                  for K in (2, 3, 4, 6, 8) for (nm, k, n) in LLAMA8B_SHAPES]

# Llama-3.1-70B MLP small-batch sweep with 1% outlier channels.
LLAMA70B_MLP = [("gate_up", 8192, 28672), ("down", 28672, 8192)]
SMALL_BATCH = [("70b_%s_m%d_K%d" % (nm, m, K), m, k, n, K, True)
               for (nm, k, n) in LLAMA70B_MLP for K in range(1, 9) for m in (1, 2, 4, 8, 16)]

# Prefill GEMM at K = 3.
PREFILL = [("70b_%s_m%d_K3" % (nm, m), m, k, n, 3, False)
           for m in (512, 2048, 8192) for (nm, k, n) in LLAMA70B_MLP]

# Llama-3.1-70B decoder-layer linear stack (attention K = 4, MLP K = 2) and
# lm_head at K = 3, at m = 1 and m = 32.
LAYER70B = [("q", 8192, 8192, 4), ("k", 8192, 1024, 4), ("v", 8192, 1024, 4),
            ("o", 8192, 8192, 4), ("gate", 8192, 28672, 2), ("up", 8192, 28672, 2),
            ("down", 28672, 8192, 2), ("lm_head", 8192, 128256, 3)]
LAYER_STACK = [("70b_layer_%s_m%d" % (nm, m), m, k, n, K, False)
               for m in (1, 32) for (nm, k, n, K) in LAYER70B]

WORKLOADS = [PR1, LLAMA8B_DECODE, SMALL_BATCH, PREFILL, LAYER_STACK]
