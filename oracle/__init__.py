"""Float64 CPU oracle of the differentiable EWA splatting path.

Test infrastructure only: imported by the tests, the package smoke check and
the benchmark's CPU baseline; never by the product library.
"""
