"""fp64 CPU oracle for the pruning path -- test infrastructure only (tests, smoke
check, benchmark CPU baseline).  Nothing on the product path imports it."""
from .pruning import *  # noqa: F401,F403
