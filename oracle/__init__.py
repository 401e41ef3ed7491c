"""CPU oracle for the AVQ-attention forward path (test infrastructure only).

``oracle.oracle`` wraps the fp64 C implementation; ``oracle.brute`` is a
separate pure-Python per-key formulation for tiny inputs. Only the tests, the
package smoke check and the benchmark's CPU-baseline leg use this package.
"""
