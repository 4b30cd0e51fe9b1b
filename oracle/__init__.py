"""Oracle: a plain, slow, obviously correct CPU restatement of the FourTune layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this package:
only the tests, the smoke check and the benchmark's CPU-baseline leg use it.  It
shares no code with the CUDA path (no kernels, headers, tables or helpers); the
two meet only in the seeded input generator, which holds none of the method's
arithmetic.

Source followed throughout: "FourTune: Towards Fully 4-Bit Efficient
Post-Training for Diffusion Models" -- §2.3 (Round(W/s) with a scale, NVFP4),
§3.1 (triple-branch pipeline), §3.2 (4-bit backward, block quantization so that
Q(G)Q(R)^T needs no requantization), §3.3 (LoRA fusion, MLP fusion) and §4.3
("Impact of Quantization Granularity": 16x16 blocks).  The pages print no
equations, so the exact format is the one the layer spec fixes: 16x16 blocks,
E2M1 codes, one E4M3 scale per block, round-to-nearest-even.

Modules
  formats  -- E2M1 / E4M3 code tables and round-to-nearest-even encoders.
  block16  -- the 16x16 block quantizer, its dequantizer, transposed packing.
  group16  -- the 1x16 group-wise quantizer with a power-of-two per-tensor
              scale (the granularity comparator of §4.3, Table 5).
  layer    -- triple-branch linear and MLP, forward and backward, float64; the
              precision variants and the 1x16 variant of the linear layer.
  stabilizer -- the truncated-SVD split W^T = S_dn S_up + R (§3.1).

Parity status: every function here is pinned by tests under tests/ (tables vs
ml_dtypes/torch, worked ties, representability, idempotence, transposed-block
equality, brute-force matmuls, adjoint and special-case identities).  What is
not pinned is the fidelity of the method as a whole (the pages' quality tables
are missing) -- "parity unpinned" for that claim only.
"""
