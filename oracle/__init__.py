"""CPU oracle for the block-sparse spatiotemporal attention path.

Test infrastructure only: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the library."""
