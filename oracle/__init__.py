"""CPU oracle for the low-rank decode path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct float64 (and, where the method fixes an
fp32 or integer pipeline, exactly emulated fp32 / integer) implementations
of what the CUDA library computes.  Only the test-suite, the package smoke
check and the benchmark's CPU-baseline leg may import this package; the
library itself never does, and there is no CPU fallback built on it.

Modules and the passages they follow:
  lowrank    truncated-SVD factorised linear y = (x A) B, its dense
             counterpart and the Eckart-Young / retained-energy quantities
             (SAES-SVD technical summary: CEALC objective and ACES RER;
             WSVD "Fine-Grained Per-Head SVD"; Swift-SVD methodology,
             covariance eigendecomposition).
  ffn        hybrid SVD / dense SwiGLU FFN with int8 RTN weights
             (LASER methodology, "Hybrid SVD-Quantization for FFNs" and
             "System Implementation").
  latent_kv  per-head latent K/V decode attention, reconstructed and
             absorbed forms (WSVD "Fine-Grained Per-Head SVD" and
             "Quantization-Aware Training (QAT) en Fused Kernel").
  w8a8       per-token int8 activation quantisation and the integer /
             fp32 W8A8 low-rank pipeline (LASER results, W8A8 setting;
             WSVD QAT section, W8A8).

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against a closed form, an identity, a library routine or brute force on
tiny inputs; none is "parity unpinned".
"""
from . import lowrank, ffn, latent_kv, w8a8  # noqa: F401
