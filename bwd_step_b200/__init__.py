"""B200 (sm_100a) forward+backward pretraining step of the nanochat-style
dense decoder, behind the C ABI of include/nanochat_b200.h."""
from .api import Model, NcError, adamw_step, launch_count  # noqa: F401
from ._lib import lib, LIB_PATH, SIGNATURES  # noqa: F401
