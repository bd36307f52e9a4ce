// gemm_sm100.cuh -- large-M W8A8 GEMM on the 5th-generation tensor cores.
//
// acc = A[m, k] * B[n, k]^T in int32 ("write-int8-quantized-kernel", Inputs:
// INT32 accumulation is mandatory; "KV-cache kernels" section 02: int8
// products accumulate in int32 and the scales are applied at the end), then
// the dequant epilogue in registers.  The pages' kernels (dp4a, a Triton
// tl.dot loop, cuBLAS/CUTLASS) are prior art; this is the sm_100a form:
//
//  - one persistent CTA per SM walks output tiles (tile = blockIdx + i*grid);
//  - warp 0 / lane 0 is the TMA producer: 128-byte-swizzled K-major tiles of
//    A (128 x 128 B) and B (BN x 128 B) into a STAGES-deep shared-memory ring,
//    completion counted in bytes on an mbarrier;
//  - warp 1 / lane 0 issues tcgen05.mma.kind::i8 (M = 128, N = BN, K = 32,
//    four per stage) into an int32 accumulator in tensor memory, and frees
//    ring slots / publishes accumulators with tcgen05.commit;
//  - epilogue warps read the accumulator with tcgen05.ld (32 lanes x 32
//    columns per instruction), apply the scales and store the outputs;
//  - per-channel mode keeps two 128 x 256 accumulators in TMEM (all 512
//    columns), so the epilogue of tile i overlaps the MMAs of tile i+1;
//  - per-group mode (group = 128 = one stage of K) keeps int32 partial
//    buffers in TMEM: the MMA writes one group's partial per buffer and moves
//    on while 16 epilogue warps convert each partial exactly to fp32 and fold
//    it in with fmaf(P_g, s[n, g], f), in ascending group order, in
//    registers.  128 x 256 tiles with two buffers when only the output is
//    wanted; 128 x 128 tiles with four buffers when the int32 sums are also
//    written.
//
// Every wait is bounded (about one second): on expiry the kernel records
// QK_ERR_TIMEOUT, every role leaves its loop, the producer waits (bounded)
// for its in-flight copies, the MMA thread waits for its in-flight MMAs, and
// the TMEM is freed before the CTA exits.
//
// The code is in gemm_core.cuh (shared pieces), gemm_1sm.cuh and
// gemm_pair.cuh (kernels) and gemm_host.cuh (plans and launches).
#pragma once

#include "gemm_host.cuh"
