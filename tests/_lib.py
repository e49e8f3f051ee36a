"""Builds libmoe.so (if stale) and imports the binding package."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def build_and_import():
    spec = importlib.util.spec_from_file_location(
        "_moe_build", os.path.join(ROOT, "fine_grained_moe_router_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import fine_grained_moe_router_b200 as M
    return M
