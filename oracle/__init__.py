"""Float64 CPU oracle for the GPTQ hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may use it.  It shares no code, tables or helpers with
the CUDA path: the two meet only through the seeded input generators in
``workloads/``.

Modules
-------
``oracle.gptq``   Hessian, damping/ordering, textbook inverse-Cholesky,
                  the column-sequential GPTQ definition and its blocked and
                  down-dated-inverse forms, packing, losses and the
                  follow-mode parity checker.
``oracle.lattice`` Independent pins: Babai's nearest-plane algorithm on the
                  Hessian lattice, brute-force CVP, round-to-nearest.
"""
