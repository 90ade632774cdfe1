"""B200-native Sketch Attention (SA) compression.

The compute path is libsa.so (CUDA, sm_100a), declared in include/sa.h; this
package holds its sources (csrc/), its build script (build.py) and a ctypes
binding (binding.py).  Importing the package does not load the library;
``SketchQuery`` does, and fails loudly if it is missing.
"""

from .binding import (  # noqa: F401
    SA_BF16,
    SA_FP32,
    ActionFusion,
    CacheKey,
    RefineParams,
    SAError,
    SketchCache,
    SketchQuery,
    WidthAdapter,
    load_library,
    mass_normalise,
    read_device_status,
    refine_layer_forward,
    refine_stack_forward,
)
