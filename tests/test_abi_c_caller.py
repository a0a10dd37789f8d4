"""The C ABI from a plain C99 program (no Python, no C++): include/csa.h compiles with
gcc -std=c99 -pedantic -Werror, the program links against libcsa.so, and the host-side
behaviour the header documents holds (tests/abi_c_caller.c).  No GPU needed."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "compressed_sparse_kv_csa_b200")


def test_plain_c_caller(tmp_path):
    import importlib.util
    spec = importlib.util.spec_from_file_location("csa_build", os.path.join(PKG, "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    exe = str(tmp_path / "abi_c_caller")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_c_caller.c"),
                           "-L", PKG, "-lcsa", "-Wl,-rpath," + PKG, "-lm", "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
