"""fp64 CPU oracle of the CODA hot path. Test infrastructure only: imported by
tests/, __graft_entry__.smoke() and bench.py's CPU baseline, never by the
library itself."""
