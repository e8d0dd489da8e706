"""Builds libdg.so before the tests load it.

The build script is loaded by file path: importing it through the package
would first run the package's __init__, which loads the library being built
(and fails when that library is missing or older than its header).
"""

import importlib.util
import os

_BUILD_PY = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                         "canvas_denoising_step_b200", "build.py")


def build_library() -> str:
    spec = importlib.util.spec_from_file_location("_libdg_build", _BUILD_PY)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()
