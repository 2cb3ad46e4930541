"""fp64 CPU oracle of the vision tower forward -- test infrastructure only (tests, smoke check,
benchmark CPU-baseline leg).  The CUDA library never imports it."""
