"""CPU oracle for SageBwd quantized attention (test infrastructure; see ``sage_oracle``)."""
from .sage_oracle import *  # noqa: F401,F403
