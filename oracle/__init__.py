"""CPU oracle for paged GQA decode attention (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline and
reference legs may import this package.  The product path never does.
"""
