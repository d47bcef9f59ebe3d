"""fp64 CPU oracle for exact attention.  Test infrastructure only (tests, smoke check, CPU baseline)."""
