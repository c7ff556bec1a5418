"""Test infrastructure only: the fp64 CPU oracle (see ``oracle.py``)."""
