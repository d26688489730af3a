"""CPU oracle of the CSA / HCA attention path — TEST INFRASTRUCTURE.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this
package.  It shares no code with the library and never imports it.
"""
from . import lc_oracle, pipeline  # noqa: F401
