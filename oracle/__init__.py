"""CPU oracle of the sigmoid-routed mixture-of-experts FFN.

Test infrastructure: only the tests, the smoke check and the benchmark's
CPU-baseline leg use it.  The product path never imports it.
"""
