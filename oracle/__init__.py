"""Independent CPU oracle for 3-D block-sparse video attention.

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the
benchmark's CPU-baseline leg may import this package; the library itself never
does, and this package never imports the library.  ``vsa_oracle`` is the
float64 NumPy oracle; ``loops`` restates it in plain Python loops for tiny
inputs.
"""
