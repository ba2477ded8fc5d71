"""CPU oracle (test infrastructure only; the product path never imports it)."""
from .aq_oracle import *  # noqa: F401,F403
from . import aq_oracle  # noqa: F401
from . import aq_paper_numerics  # noqa: F401
