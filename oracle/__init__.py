"""CPU oracle of the sparsely-gated MoE layer forward (test infrastructure only).

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this
package; the CUDA library never does.
"""
