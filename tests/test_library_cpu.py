"""The C-ABI library on a host without a GPU: it builds, loads, exports every
symbol include/ln.h declares, and rejects bad arguments before it makes any
CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ln.h")


@pytest.fixture(scope="module")
def lib():
    from layernorm_fwd_bwd_b200 import build
    build.build()
    from layernorm_fwd_bwd_b200 import ln
    return ln


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ln_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("ln_forward", "ln_backward", "ln_status_string", "ln_launch_count",
              "ln_version"):
        assert n in names


def test_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.library_path())
    for name in declared_functions():
        assert hasattr(so, name), f"{name} not exported"
    dyn = subprocess.run(["nm", "-D", "--defined-only", lib.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ln_[a-z_0-9]+)$", dyn, flags=re.M))
    assert set(declared_functions()) <= exported


def test_status_strings(lib):
    names = ["LN_OK", "LN_ERR_NULL", "LN_ERR_SHAPE", "LN_ERR_DTYPE", "LN_ERR_EPS",
             "LN_ERR_WORKSPACE", "LN_ERR_CUDA", "LN_ERR_SCRATCH", "LN_ERR_FLAGS",
             "LN_ERR_ALIAS"]
    for code, name in enumerate(names):
        assert lib.ln_status_string(code).startswith(name)
        assert getattr(lib, name) == code
    assert lib.ln_status_string(99) == "unknown ln_status"
    assert lib.version() == 3


def test_host_validation_without_gpu(lib):
    # Each of these returns before the library touches the CUDA runtime.
    f = lib.raw_forward
    nz = 16  # any non-NULL address: never dereferenced on these paths
    n0 = lib.launch_count()   # per process: GPU tests may have run before
    assert f(nz, nz, nz, nz, nz, nz, -1, 8, 1e-5, 0, None) == lib.LN_ERR_SHAPE
    assert f(nz, nz, nz, nz, nz, nz, 4, 0, 1e-5, 0, None) == lib.LN_ERR_SHAPE
    assert f(nz, nz, nz, nz, nz, nz, 4, (1 << 24) + 1, 1e-5, 0, None) == lib.LN_ERR_SHAPE
    assert f(nz, nz, nz, nz, nz, nz, 4, 8, 1e-5, 3, None) == lib.LN_ERR_DTYPE
    assert f(nz, nz, nz, nz, nz, nz, 4, 8, 0.0, 0, None) == lib.LN_ERR_EPS
    assert f(nz, nz, nz, nz, nz, nz, 4, 8, float("nan"), 0, None) == lib.LN_ERR_EPS
    assert f(nz, nz, nz, nz, nz, nz, 4, 8, float("inf"), 1, None) == lib.LN_ERR_EPS
    assert f(nz, nz, nz, nz, nz, nz, 4, 8, -1e-5, 1, None) == lib.LN_ERR_EPS
    assert f(None, nz, nz, nz, nz, nz, 4, 8, 1e-5, 0, None) == lib.LN_ERR_NULL
    assert f(nz, nz, nz, nz, nz, None, 4, 8, 1e-5, 0, None) == lib.LN_ERR_NULL
    assert f(None, None, None, None, None, None, 0, 8, 1e-5, 0, None) == lib.LN_OK
    b = lib.raw_backward
    assert b(nz, nz, nz, nz, nz, nz, nz, nz, -1, 8, 0, None) == lib.LN_ERR_SHAPE
    assert b(nz, nz, nz, nz, nz, nz, nz, nz, 4, 8, 7, None) == lib.LN_ERR_DTYPE
    assert b(nz, None, nz, nz, nz, nz, nz, nz, 4, 8, 0, None) == lib.LN_ERR_NULL
    assert b(nz, nz, None, nz, nz, nz, nz, nz, 0, 8, 0, None) == lib.LN_ERR_NULL
    assert lib.launch_count() == n0


def test_variant_validation_without_gpu(lib):
    # ln_forward_residual and ln_backward_ex validate like the plain calls,
    # plus their own arguments, before any CUDA call.
    nz = 16
    n0 = lib.launch_count()
    r = lib.raw_forward_residual
    assert r(nz, nz, nz, nz, nz, nz, nz, nz, -1, 8, 1e-5, 0, None) == lib.LN_ERR_SHAPE
    assert r(nz, nz, nz, nz, nz, nz, nz, nz, 4, 8, 1e-5, 5, None) == lib.LN_ERR_DTYPE
    assert r(nz, nz, nz, nz, nz, nz, nz, nz, 4, 8, 0.0, 0, None) == lib.LN_ERR_EPS
    assert r(None, nz, nz, nz, nz, nz, nz, nz, 4, 8, 1e-5, 0, None) == lib.LN_ERR_NULL
    assert r(nz, nz, nz, nz, nz, None, nz, nz, 4, 8, 1e-5, 0, None) == lib.LN_ERR_NULL
    assert r(nz, None, nz, nz, nz, nz, nz, nz, 4, 8, 1e-5, 1, None) == lib.LN_ERR_NULL
    assert r(None, None, None, None, None, None, None, None, 0, 8, 1e-5, 0, None) == lib.LN_OK
    x = lib.raw_backward_ex
    acc = lib.LN_BWD_ACCUMULATE_DINP | lib.LN_BWD_ACCUMULATE_DPARAMS
    rec = lib.LN_BWD_RECOMPUTE_STATS
    assert x(nz, nz, nz, nz, nz, nz, nz, nz, -1, 8, 1e-5, 0, 0, None) == lib.LN_ERR_SHAPE
    assert x(nz, nz, nz, nz, nz, nz, nz, nz, 4, 8, 1e-5, 3, 0, None) == lib.LN_ERR_DTYPE
    assert x(nz, nz, nz, nz, nz, nz, nz, nz, 4, 8, 1e-5, 0, 8, None) == lib.LN_ERR_FLAGS
    assert x(nz, nz, nz, nz, nz, nz, nz, nz, 4, 8, 1e-5, 0, 1 << 31, None) == lib.LN_ERR_FLAGS
    # eps is checked only when the statistics are recomputed
    assert x(nz, nz, nz, nz, nz, nz, nz, nz, 4, 8, 0.0, 0, rec, None) == lib.LN_ERR_EPS
    assert x(nz, nz, nz, nz, nz, nz, nz, nz, 4, 8, float("nan"), 1, rec | acc,
             None) == lib.LN_ERR_EPS
    # mean/rstd are required unless recomputed
    assert x(nz, nz, nz, nz, nz, nz, None, nz, 4, 8, 1e-5, 0, acc, None) == lib.LN_ERR_NULL
    assert x(nz, nz, nz, nz, nz, nz, nz, None, 4, 8, 1e-5, 0, 0, None) == lib.LN_ERR_NULL
    assert x(nz, None, nz, nz, nz, nz, nz, nz, 4, 8, 1e-5, 0, rec, None) == lib.LN_ERR_NULL
    # N == 0 with accumulated parameters has nothing to do (no memset either)
    assert x(None, nz, nz, None, None, None, None, None, 0, 8, 0.0, 0,
             lib.LN_BWD_ACCUMULATE_DPARAMS, None) == lib.LN_OK
    assert lib.launch_count() == n0


def test_overlapping_outputs_are_refused_without_gpu(lib):
    """Outputs that overlap inputs where the header forbids it return
    LN_ERR_ALIAS before any CUDA call (addresses are never dereferenced; every
    case here is refused on the host, so none can reach a device)."""
    n0 = lib.launch_count()
    N, C = 4, 8
    act = N * C * 2                      # bytes of one bf16 activation array
    a, b, c, d = 1 << 20, 2 << 20, 3 << 20, 4 << 20   # disjoint fake device addresses
    f = lib.raw_forward
    assert f(a, b, b + 64, a, c, d, N, C, 1e-5, 1, None) == lib.LN_ERR_ALIAS       # out == inp
    assert f(a, b, b + 64, a + act - 2, c, d, N, C, 1e-5, 1, None) == lib.LN_ERR_ALIAS
    r = lib.raw_forward_residual
    assert r(a, b, c, c + 64, a, d, c + 128, c + 256, N, C, 1e-5, 1, None) == lib.LN_ERR_ALIAS
    assert r(a, b, c, c + 64, d, b + 2, c + 128, c + 256, N, C, 1e-5, 1, None) == lib.LN_ERR_ALIAS
    assert r(a, a + 16, c, c + 64, d, d + act, c + 128, c + 256, N, C, 1e-5, 1,
             None) == lib.LN_ERR_ALIAS                                               # outputs
    bw = lib.raw_backward
    assert bw(a, c, c + 64, a, b, d, c + 128, c + 256, N, C, 1, None) == lib.LN_ERR_ALIAS
    assert bw(a, c, c + 64, b, a + 8, d, c + 128, c + 256, N, C, 1, None) == lib.LN_ERR_ALIAS
    x = lib.raw_backward_ex
    assert x(a, c, c + 64, a, b, d, None, None, N, C, 1e-5, 1, lib.LN_BWD_RECOMPUTE_STATS,
             None) == lib.LN_ERR_ALIAS
    assert lib.launch_count() == n0


def test_every_output_overlap_is_refused_without_gpu(lib):
    """No output may share a byte with another output or with any array the
    call reads: the statistics, the parameter gradients and the small arrays
    included.  Each case starts from a layout of disjoint fake addresses and
    moves one array onto another; all are refused on the host."""
    n0 = lib.launch_count()
    N, C = 4, 8
    act, par, stat, grad = N * C * 2, C * 2, N * 4, C * 4     # bf16 sizes in bytes
    base = 1 << 20
    fwd = dict(out=base, mean=2 * base, rstd=3 * base, inp=4 * base, weight=5 * base,
               bias=6 * base)

    def f(**moved):
        p = {**fwd, **moved}
        return lib.raw_forward(p["out"], p["mean"], p["rstd"], p["inp"], p["weight"],
                               p["bias"], N, C, 1e-5, 1, None)

    for moved in (dict(rstd=fwd["mean"]),                    # mean == rstd
                  dict(rstd=fwd["mean"] + stat - 4),         # last float shared
                  dict(mean=fwd["out"] + act - 4),           # mean inside out's tail
                  dict(out=fwd["rstd"] + 4),                 # out over rstd
                  dict(mean=fwd["weight"] + par - 2),        # mean over weight's last element
                  dict(rstd=fwd["bias"]),
                  dict(mean=fwd["inp"] + 2 * C)):
        assert f(**moved) == lib.LN_ERR_ALIAS, moved

    res = dict(fwd, resid_out=7 * base, branch=8 * base)

    def r(**moved):
        p = {**res, **moved}
        return lib.raw_forward_residual(p["resid_out"], p["out"], p["mean"], p["rstd"],
                                        p["inp"], p["branch"], p["weight"], p["bias"], N, C,
                                        1e-5, 1, None)

    for moved in (dict(mean=res["resid_out"] + 8), dict(resid_out=res["weight"]),
                  dict(rstd=res["branch"] + act - 4), dict(out=res["branch"])):
        assert r(**moved) == lib.LN_ERR_ALIAS, moved

    bwd = dict(dinp=base, dweight=2 * base, dbias=3 * base, dout=4 * base, inp=5 * base,
               weight=6 * base, mean=7 * base, rstd=8 * base)

    def b(flags=0, **moved):
        p = {**bwd, **moved}
        return lib.raw_backward_ex(p["dinp"], p["dweight"], p["dbias"], p["dout"], p["inp"],
                                   p["weight"], p["mean"], p["rstd"], N, C, 1e-5, 1, flags,
                                   None)

    acc = lib.LN_BWD_ACCUMULATE_DINP | lib.LN_BWD_ACCUMULATE_DPARAMS
    for flags in (0, acc):
        for moved in (dict(dbias=bwd["dweight"]),                 # dweight == dbias
                      dict(dbias=bwd["dweight"] + grad - 4),
                      dict(dweight=bwd["weight"]),                # dweight over weight
                      dict(dbias=bwd["mean"] + stat - 4),         # dbias over mean's tail
                      dict(dweight=bwd["rstd"]),
                      dict(dweight=bwd["inp"] + act - 4),
                      dict(dbias=bwd["dinp"] + 16),               # over another output
                      dict(dinp=bwd["weight"] - act + 2)):        # dinp's tail over weight
            assert b(flags, **moved) == lib.LN_ERR_ALIAS, (flags, moved)
    # the plain and no-alloc entry points share the checks
    p = dict(bwd, dbias=bwd["dweight"])
    assert lib.raw_backward(p["dinp"], p["dweight"], p["dbias"], p["dout"], p["inp"],
                            p["weight"], p["mean"], p["rstd"], N, C, 1, None) == lib.LN_ERR_ALIAS
    import torch
    if not torch.cuda.is_available():
        # without a device the no-alloc call stops at its device lookup,
        # before the shared checks; with one it reaches them
        pytest.skip("ln_backward_noalloc reaches the shared checks only with a device")
    with pytest.raises(lib.LNError) as e:
        lib.ln_backward_noalloc(p["dinp"], p["dweight"], p["dbias"], p["dout"], p["inp"],
                                p["weight"], p["mean"], p["rstd"], N, C, lib.LN_BF16)
    assert e.value.status == lib.LN_ERR_ALIAS
    assert lib.launch_count() == n0


def test_binding_raises_lnerror(lib):
    with pytest.raises(lib.LNError) as e:
        lib.ln_forward(16, 16, 16, 16, 16, 16, -3, 8, 1e-5, 0, stream=0)
    assert e.value.status == lib.LN_ERR_SHAPE


def test_rejects_oversized_products(lib):
    nz = 16
    assert lib.raw_forward(nz, nz, nz, nz, nz, nz, 1 << 40, 1 << 11, 1e-5, 0,
                           None) == lib.LN_ERR_SHAPE
    assert lib.raw_backward(nz, nz, nz, nz, nz, nz, nz, nz, 1 << 30, 1 << 21, 1,
                            None) == lib.LN_ERR_SHAPE


def test_tolerance_helpers():
    import numpy as np

    import tolerances as tol
    ref = np.array([1.0, -2.0, 0.5])
    assert tol.max_ulps(ref, ref) == 0.0
    # one bf16 ulp at 1.0 is 2^-7
    assert tol.max_ulps(ref + np.array([2.0 ** -7, 0, 0]), ref) == 1.0
    # near-zero values are judged at 2^-8 * max|ref|
    assert tol.max_ulps(np.array([2.0 ** -15, 1.0]), np.array([0.0, 1.0])) == 1.0
    assert tol.rel_max(ref * (1 + 1e-6), ref) <= 1.1e-6
    assert tol.rel_max(np.array([1e-3 + 1e-8]), np.array([1e-3]), scale=1.0) <= 1.1e-8
    with pytest.raises(AssertionError):
        tol.check("x", ref * (1 + 1e-4), ref, "f32", "act_fwd")
    # one fp16 ulp at 1.0 is 2^-10; below 2^-14 the spacing stays 2^-24
    assert tol.max_ulps(ref + np.array([2.0 ** -10, 0, 0]), ref, dtype="f16") == 1.0
    assert tol.max_ulps(np.array([2.0 ** -24]), np.array([0.0]), dtype="f16") == 1.0
    tol.check("x", ref + np.array([2.0 ** -9, 0, 0]), ref, "f16", "act_fwd")
    with pytest.raises(AssertionError):
        tol.check("x", ref + np.array([2.0 ** -8 * 1.01, 0, 0]), ref, "f16", "act_fwd")


def test_package_forwards_the_binding(lib):
    """Every public name of the binding is reachable from the package."""
    import layernorm_fwd_bwd_b200 as pkg
    public = [n for n in vars(lib) if not n.startswith("_") and (
        n.startswith(("ln_", "LN_", "raw_")) or n in pkg._BINDING_NAMES)]
    for n in ("ln_forward_residual", "ln_backward_ex", "ln_backward_noalloc", "LN_F16",
              "LN_BWD_RECOMPUTE_STATS", "device_status"):
        assert n in public
    for n in public:
        assert getattr(pkg, n) is getattr(lib, n), n
    with pytest.raises(AttributeError):
        pkg.ln_no_such_entry
    with pytest.raises(AttributeError):
        pkg.no_such_name


def test_binding_constants_match_the_header(lib):
    """Every LN_* constant of the binding has the value include/ln.h gives it,
    read by compiling a small C program against the header."""
    from layernorm_fwd_bwd_b200 import build
    names = sorted(n for n in vars(lib) if n.startswith("LN_"))
    assert {"LN_MAX_C", "LN_F16", "LN_ERR_ALIAS", "LN_BWD_RECOMPUTE_STATS"} <= set(names)
    prints = "".join(f'printf("{n} %lld\\n", (long long)({n}));' for n in names)
    src = f"#include <stdio.h>\n#include \"ln.h\"\nint main(void) {{ {prints} return 0; }}\n"
    os.makedirs(build.BUILD_DIR, exist_ok=True)
    exe = os.path.join(build.BUILD_DIR, "ln_header_constants")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-x", "c", "-", "-o", exe], input=src, text=True, check=True)
    got = dict(line.split() for line in
               subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
               if line)
    assert {n: int(v) for n, v in got.items()} == {n: getattr(lib, n) for n in names}


# C parameter types of include/ln.h and the ctypes type the binding must
# declare for each
_CTYPES = {"void *": "c_void_p", "const void *": "c_void_p", "float *": "c_void_p",
           "const float *": "c_void_p", "int64_t": "c_long", "int": "c_int",
           "float": "c_float", "unsigned int": "c_uint", "ln_stream_t": "c_void_p",
           "unsigned int *": "LP_c_uint", "void": None}


def _prototypes():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for ret, name, params in re.findall(
            r"^\s*(int|const char \*|uint64_t)\s*(ln_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M):
        types = []
        for p in params.split(","):
            p = " ".join(p.split())
            if p in ("void", ""):
                continue
            t = re.sub(r"\s*\b\w+$", "", p)          # drop the parameter name
            types.append(re.sub(r"\s*\*", " *", t).strip())
        out[name] = (ret, types)
    return out


_RESTYPES = {"int": "c_int", "const char *": "c_char_p", "uint64_t": "c_ulong"}


def test_binding_signatures_match_the_header(lib):
    """Every function of include/ln.h is declared to ctypes with the same
    number of parameters and matching types, so no call passes an argument
    the library reads as something else."""
    protos = _prototypes()
    assert set(protos) == set(declared_functions())
    for name, (ret, types) in protos.items():
        fn = getattr(lib._lib, name)
        got = [t.__name__ for t in (fn.argtypes or [])]
        want = [_CTYPES[t] for t in types]
        # ctypes spells the 64-bit integers c_long / c_ulong on LP64 hosts
        got = ["c_long" if g in ("c_int64", "c_longlong") else g for g in got]
        assert got == want, f"{name}: header {types}, binding {got}"
        res = {"c_uint64": "c_ulong", "c_ulonglong": "c_ulong"}.get(fn.restype.__name__,
                                                                     fn.restype.__name__)
        assert res == _RESTYPES[ret], f"{name}: returns {ret}, binding {fn.restype.__name__}"


def test_header_compiles_as_cpp():
    """C++ callers include the same header (extern "C", no warnings)."""
    src = ('#include "ln.h"\n'
           'int (*const version)(void) = ln_version;\n'
           'int main() { return version != ln_version; }\n')
    subprocess.run(["g++", "-std=c++11", "-Wall", "-Werror", "-pedantic", "-I",
                    os.path.join(ROOT, "include"), "-x", "c++", "-", "-fsyntax-only"],
                   input=src, text=True, check=True)


def test_workspace_limit_and_last_cuda_error_on_host(lib):
    """ln_set_workspace_limit refuses a negative cap before touching CUDA;
    without a usable device it returns LN_ERR_CUDA, and ln_last_cuda_error
    then names the runtime call that failed."""
    import torch
    assert lib._lib.ln_set_workspace_limit(-1) == lib.LN_ERR_SHAPE
    assert isinstance(lib.last_cuda_error(), str) and lib.last_cuda_error()
    if torch.cuda.is_available():
        pytest.skip("a device is present: the failing path is not reachable here")
    assert lib._lib.ln_set_workspace_limit(0) == lib.LN_ERR_CUDA
    text = lib.last_cuda_error()
    assert "cudaGetDevice" in text and text.startswith("cuda"), text
    with pytest.raises(lib.LNError) as e:
        lib.set_workspace_limit(0)
    assert "cudaGetDevice" in str(e.value)


def _code(path):
    """C++ source with comments and string literals removed."""
    text = open(path).read()
    text = re.sub(r"//[^\n]*", "", text)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r'"(?:\\.|[^"\\])*"', '""', text)


def test_only_the_pooled_backward_creates_the_pool():
    """ln_backward_noalloc must not create the library's memory pool: the
    pool is created in one function (workspace_pool), which is reached only
    from the branch of the backward that has no caller-provided scratch."""
    csrc = os.path.join(ROOT, "layernorm_fwd_bwd_b200", "csrc")
    creators, callers = [], []
    for f in sorted(os.listdir(csrc)):
        code = _code(os.path.join(csrc, f))
        if "cudaMemPoolCreate" in code:
            creators.append(f)
        for m in re.finditer(r"\bworkspace_pool\s*\(", code):
            callers.append((f, code[:m.start()]))
    assert creators == ["ln_api.cu"]
    api = _code(os.path.join(csrc, "ln_api.cu"))
    body = api[api.index("cudaError_t workspace_pool("):]
    body = body[:body.index("\n}\n")]
    assert "cudaMemPoolCreate" in body
    assert api.count("cudaMemPoolCreate") == 1
    uses = [(f, pre) for f, pre in callers
            if not re.search(r"cudaError_t\s+$", pre)]   # skip declarations/definition
    assert [f for f, _ in uses] == ["ln_dispatch.cuh"], uses
    pre = uses[0][1]
    branch = pre[pre.rindex("float *partial = a.scratch;"):]
    assert re.search(r"if\s*\(\s*!\s*partial\s*\)\s*\{", branch), branch[-300:]
