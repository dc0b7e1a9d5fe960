"""B200-native (sm_100a) 1-bit Adam compressed-phase step.

The product is the C-ABI library ``libonebit.so`` (include/onebit.h); this
package holds its CUDA sources (``csrc/``), the build script, the ctypes
binding with the C names (``_lib``) and a small optimizer object over it
(``OneBitAdam``).  Importing the package loads the library and fails loudly
when it has not been built.
"""

from . import _lib
from ._lib import (  # noqa: F401
    OB_ADAM, OB_BF16, OB_ECUDA, OB_EINVAL, OB_ENOMEM, OB_EPHASE, OB_F32, OB_LAMB, OB_OK,
    OB_RULE_MOMENTUM_ERROR, OB_RULE_SCALED_SIGN, OB_RULE_TWO_BIT, OB_STATUS_NONFINITE, OneBitError, make_config, ob_compress, ob_create, ob_destroy,
    ob_get_status, ob_get_step, ob_layout, ob_refresh_step, ob_server_reduce, ob_set_step,
    ob_step, ob_step_host, ob_warmup_step,
)

_lib.load()

from .optimizer import OneBitAdam  # noqa: E402,F401
