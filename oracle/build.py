"""Compile the oracle's C parts (test infrastructure) into oracle/liboracle_patches.so
(great-circle FPS, patch tables, pooling, scores, top R) and oracle/liboracle_mesh.so
(geodesic FPS on a mesh graph)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "patches.c")
LIB = os.path.join(HERE, "liboracle_patches.so")
MESH_SRC = os.path.join(HERE, "mesh.c")
MESH_LIB = os.path.join(HERE, "liboracle_mesh.so")


def _compile(src: str, lib: str, force: bool) -> str:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(src):
        return lib
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC",
           "-shared", src, "-o", lib + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False) -> str:
    _compile(MESH_SRC, MESH_LIB, force)
    return _compile(SRC, LIB, force)


def build_mesh(force: bool = False) -> str:
    return _compile(MESH_SRC, MESH_LIB, force)


if __name__ == "__main__":
    print(build(force=True))
