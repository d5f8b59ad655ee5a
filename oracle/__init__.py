"""Test infrastructure: the fp64 CPU oracle for the RSM mixer. Not part of the product path."""
