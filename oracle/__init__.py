"""Test infrastructure: the fp64 CPU oracle.  Never imported by the library."""
