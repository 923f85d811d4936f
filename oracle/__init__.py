"""CPU oracle for the CSA layer — test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference leg may import this
package.  The CUDA library and its Python binding never import it; the two share no code.
Pins: tests/test_oracle_formats.py and tests/test_oracle_layer.py.  End-to-end parity against the
pages is unpinned (they print no worked example for the layer); every stage is pinned by closed
forms, library routines, brute force and invariants.
"""
