"""B200-native (sm_100a) VDN-H3 dual-branch hybrid attention.

The compute path is the C-ABI library ``libvdnattn.so`` (hand-written CUDA
for sm_100a) built in-tree next to this file; :mod:`.binding` marshals
arguments to it.  Importing the package does not load the library; the first
call that needs it does, and fails loudly if it is missing.
"""
from .workloads import WORKLOADS, BY_NAME, Workload, make_inputs  # noqa: F401
