"""The oracle: a plain fp64 CPU restatement of PISA selection and attention.

Test infrastructure only: the tests, the smoke check and the benchmark's CPU
baseline use it; the product library never does.
"""
from .oracle import *  # noqa: F401,F403
