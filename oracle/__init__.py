"""Float64 CPU oracle of the WTConv layer -- test infrastructure only.

Imported by the tests, the smoke check and the benchmark's CPU-baseline leg;
never by the library.
"""
from .wtconv_oracle import (  # noqa: F401
    BANDS, SIGN, haar_analysis, haar_synthesis, dwconv, dwcorr_weight,
    forward, backward, analysis_closed_form, synthesis_closed_form, level_outputs,
)
