"""CPU oracle for the Atom W4A4 hot path -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package. The CUDA library never does.

`oracle.c_oracle` wraps the plain C oracle (`atom_oracle.c`);
`oracle.numpy_oracle` is an independent numpy restatement used to cross-check
it bit for bit.
"""
