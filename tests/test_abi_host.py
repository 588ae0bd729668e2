"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

* libcsa.so builds for sm_100a, loads, and exports every function that
  include/csa.h declares.
* Host validation returns the documented status codes.  These cases run in
  a subprocess with CUDA_VISIBLE_DEVICES="" so that no device is reachable
  even if a validation bug let a call through.
"""

import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# csa_index_topk workspace for 2 queries over 32768 entries (fp32 scores):
# the scores, then the cleared region (per query a 4096-bin histogram, a tie
# count padded to 16 bytes over the batch, a 256-bin second-level
# histogram), each rounded up to 256 bytes
_INDEX_WS_2x32768 = 2 * 32768 * 4 + ((2 * 4096 * 4 + 16 + 2 * 256 * 4 + 255) // 256) * 256


def _declared():
    src = open(os.path.join(ROOT, "include", "csa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:csa_status|size_t|const char\*)\s+(\w+)\s*\(", src, flags=re.M)))


def test_build_and_exports():
    from long_context_sparse_gated_b200 import build
    lib_path = build.build()
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True).stdout
    syms = set(l.split()[-1] for l in out.splitlines() if l.strip())
    decl = _declared()
    assert len(decl) >= 9
    missing = [d for d in decl if d not in syms]
    assert not missing, f"declared but not exported: {missing}"
    import long_context_sparse_gated_b200 as m
    assert set(m.EXPORTS) <= set(decl)


_VALIDATION = r"""
import ctypes, sys
sys.path.insert(0, ROOT)
import long_context_sparse_gated_b200 as m
L = m.lib()
P = m.make_params(B=2, d=512, r=64, m=4, n_idx_heads=64, idx_dim=128, topk=512, n_heads=64,
                  window=128, softmax_scale=0.044)
A = 0x10000  # a fake, 16-byte aligned address; every case below fails validation first
kv = m.CsaKv(A, A, 100)
def st(name, *args):
    return getattr(L, name)(*args)
r = {}
r['null_params'] = st('csa_index_topk', None, A, A, A, A, A, 100, A, 1, 10, A, A, 1 << 20, None, None)
bad = m.make_params(B=2, d=256, r=64, m=4)
r['bad_d'] = st('csa_compress', ctypes.byref(bad), A, A, A, 8, A, A, A, 1, None, kv, None, None, None)
r['misaligned'] = st('csa_compress', ctypes.byref(P), A + 4, A, A, 8, A, A, A, 1, None, kv, None, None, None)
r['small_ws'] = st('csa_index_topk', ctypes.byref(P), A, A, A, A, A, 100, A, 1, 100, A, A, 16, None, None)
r['k_too_big'] = st('csa_index_topk', ctypes.byref(m.make_params(B=2, d=512, r=64, m=4, n_idx_heads=64, idx_dim=128, topk=4096)), A, A, A, A, A, 100, A, 1, 10, A, A, 1 << 20, None, None)
r['n_max_gt_cap'] = st('csa_index_topk', ctypes.byref(P), A, A, A, A, A, 100, A, 1, 101, A, A, 1 << 30, None, None)
r['null_sink'] = st('csa_sparse_attn', ctypes.byref(P), A, kv, A, m.CsaKv(A, A, 128), None, A, 1, A, A, 1 << 30, None, None)
r['small_window'] = st('csa_sparse_attn', ctypes.byref(P), A, kv, A, m.CsaKv(A, A, 64), A, A, 1, A, A, 1 << 30, None, None)
state_small = m.CsaState(m.CsaKv(A, A, 256), A, A, A, 8)      # s_cap 8 < T + 2m
r['state_small_ring'] = st('csa_state_append', ctypes.byref(P), A, A, A, A, A, 1, state_small, kv, None, None, None, None)
state_ok = m.CsaState(m.CsaKv(A, A, 256), A, A, A, 64)
ck_bad = m.CsaCkpt(A, A, A, A, A, 2, 1022)                       # period not a multiple of m
r['ckpt_period'] = st('csa_state_append', ctypes.byref(P), A, A, A, A, A, 1, state_ok, kv, None, ctypes.byref(ck_bad), None, None)
r['restore_null'] = st('csa_state_restore', ctypes.byref(P), A, None, state_ok, None, None)
r['quant_dim'] = st('csa_index_quantize', ctypes.byref(m.make_params(B=1, d=512, r=64, m=4, idx_dim=96)), A, 8, A, A, None)
r['ikc_rope'] = st('csa_index_compress', ctypes.byref(P), A, A, A, 8, A, A, A, 1, 6, None, A, A, 10, None, None)
r['ws_bytes'] = L.csa_index_topk_workspace_bytes(ctypes.byref(P), 1, 32768)
r['attn_ws'] = L.csa_sparse_attn_workspace_bytes(ctypes.byref(P), 1)
r['name'] = L.csa_status_string(-4).decode()
print(repr(r))
"""


def test_host_validation_codes():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    code = "ROOT = %r\n" % ROOT + _VALIDATION
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr
    r = eval(out.stdout.strip().splitlines()[-1])
    assert r["null_params"] == -1
    assert r["bad_d"] == -2
    assert r["misaligned"] == -3
    assert r["small_ws"] == -4
    assert r["k_too_big"] == -2
    assert r["n_max_gt_cap"] == -1
    assert r["null_sink"] == -1
    assert r["small_window"] == -1
    assert r["state_small_ring"] == -1
    assert r["ckpt_period"] == -1
    assert r["restore_null"] == -1
    assert r["quant_dim"] == -2
    assert r["ikc_rope"] == -2
    assert r["ws_bytes"] == _INDEX_WS_2x32768
    assert r["attn_ws"] > 0
    assert r["name"] == "CSA_ERR_WORKSPACE"


def test_plain_c_client_compiles_links_and_validates(tmp_path):
    """The header is a C99 header: a C program builds against it alone,
    links libcsa.so and gets the documented status codes."""
    import shutil
    from long_context_sparse_gated_b200 import build
    lib_path = build.build()
    cc = shutil.which("gcc") or shutil.which("cc")
    assert cc, "no C compiler"
    exe = tmp_path / "abi_c_client"
    libdir = os.path.dirname(lib_path)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "abi_c_client.c"), "-L", libdir, "-l:" + os.path.basename(lib_path),
                        "-Wl,-rpath," + libdir, "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([str(exe)], capture_output=True, text=True, env=env, timeout=120)
    assert out.returncode == 0, out.stderr
    s_null, s_bad, s_align, ws, name = out.stdout.split()
    assert (int(s_null), int(s_bad), int(s_align)) == (-1, -2, -3)
    assert int(ws) == _INDEX_WS_2x32768
    assert name == "CSA_ERR_ALIGN"
