"""Randomly perturbed argument structs against the host-side checks of every entry point
(no GPU): each call returns one of the documented status codes and never crashes the
process. Each struct starts from a valid call and has up to three fields replaced by
extreme or malformed values. Pointers are NULL, a misaligned address or an aligned address
that is never dereferenced on the host. The child process sees no GPU (it runs with
CUDA_VISIBLE_DEVICES empty, also on a GPU machine), so a call that passes every check
stops at its first device query with CSA_ERR_CUDA and no kernel ever receives these
pointers. A crash of the child fails the test instead of the test run."""

import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import ctypes as C, sys
import numpy as np
sys.path.insert(0, {root!r})
import long_context_compressed_layer_b200 as csa
L = csa.lib()
rng = np.random.default_rng({seed})
F, MISALIGNED = 1 << 20, (1 << 20) + 4
OK = {{csa.CSA_OK, csa.CSA_ERR_INVALID_ARG, csa.CSA_ERR_UNSUPPORTED, csa.CSA_ERR_WORKSPACE,
      csa.CSA_ERR_CUDA}}
INTS = [-1, 0, 1, 2, 3, 4, 16, 63, 64, 127, 128, 129, 1000, 1024, 2048, 4096, 65535, 65536,
        1 << 20, 1 << 30, (1 << 31) - 1, -(1 << 31)]
WS = 1 << 40  # a workspace size no check refuses

BASES = [
    (lambda: csa.CompressArgs(1, 64, 4, 1, 0, 10000.0, 1e-6, F, F, F, F, F, None, None, None,
                              F, F, 128, None),
     lambda a: L.csa_compress(C.byref(a), None)),
    (lambda: csa.IkeyArgs(1, 64, 4, 1, 0, F, F, F, F, F, None, None, F, F, 128, None),
     lambda a: L.csa_compress_index_keys(C.byref(a), None)),
    (lambda: csa.AppendArgs(2, 4, 1, 10000.0, 1e-6, *([F] * 6), None, *([F] * 7), 128, F,
                            *([None] * 11), None),
     lambda a: L.csa_decode_append(C.byref(a), None)),
    (lambda: csa.IqueryArgs(16, 1536, 64, F, F, F, F, None, None),
     lambda a: L.csa_indexer_query(C.byref(a), None)),
    (lambda: csa.OprojArgs(64, 128, 16, 1024, 7168, F, F, F, F, None),
     lambda a: L.csa_grouped_out_proj(C.byref(a), F, WS, None)),
    (lambda: csa.TopkArgs(2, 64, 512, 1024, F, F, F, F, F, F, F, None, None),
     lambda a: L.csa_indexer_topk(C.byref(a), F, WS, None)),
    (lambda: csa.TopkArgs(2, 64, 512, 1024, F, F, F, F, F, F, F, None, None),
     lambda a: L.csa_indexer_topk_bf16(C.byref(a), F, WS, None)),
    (lambda: csa.AttnArgs(2, 128, 1024, 4096, F, F, F, F, F, F, F, F, 0.0, 10000.0, 1, F,
                          None, None),
     lambda a: L.csa_sparse_attn_decode(C.byref(a), F, WS, None)),
    (lambda: csa.AttnArgs(2, 128, 1024, 4096, F, F, F, F, F, F, F, F, 0.0, 10000.0, 1, F,
                          None, None),
     lambda a: L.hca_attn_decode(C.byref(a), F, WS, None)),
    (lambda: csa.AttnArgs(2, 128, 1024, 4096, F, F, F, F, F, F, F, F, 0.0, 10000.0, 1, F,
                          None, None),
     lambda a: L.csa_sparse_attn_decode_noalloc(C.byref(a), None)),
    (lambda: csa.PrefillArgs(4096, 300, 4, 128, 64, 1024, 1152, 0.0, 10000.0, 1e-6, 1, 0,
                             *([F] * 5), None, F, F, *([F] * 10), F, None, None, None),
     lambda a: L.csa_prefill(C.byref(a), F, WS, None)),
]


def mutate(a, count):
    fields = type(a)._fields_
    for i in rng.choice(len(fields), size=count, replace=False):
        name, ty = fields[i]
        if ty is C.c_void_p:
            setattr(a, name, [None, F, MISALIGNED][rng.integers(3)])
        elif ty is csa.Pages:  # a paged-cache descriptor: table and sizes perturbed together
            setattr(a, name, csa.Pages([None, F, MISALIGNED][rng.integers(3)],
                                       int(rng.choice(INTS)), int(rng.choice(INTS)),
                                       int(rng.choice(INTS))))
        elif ty is C.c_float:
            setattr(a, name, float(rng.choice([-1.0, 0.0, 1e-6, 0.0442, 1.0, 1e4, np.nan])))
        elif ty is C.c_int64:
            setattr(a, name, int(rng.choice(INTS + [1 << 40, -(1 << 40)])))
        else:
            setattr(a, name, int(rng.choice(INTS)))
    return a


seen = {{}}
for i in range({n}):
    make, call = BASES[i % len(BASES)]
    a = mutate(make(), int(rng.integers(0, 4)))
    st = call(a)
    assert st in OK, (type(a).__name__, st)
    seen[st] = seen.get(st, 0) + 1
for fn, nargs in ((L.csa_indexer_topk_workspace_size, 3), (L.csa_attn_workspace_size, 3),
                  (L.csa_prefill_workspace_size, 4),
                  (L.csa_grouped_out_proj_workspace_size, 3)):
    for _ in range(200):
        fn(*[int(rng.choice(INTS)) for _ in range(nargs)])
print(sorted(seen.items()))
"""


def test_perturbed_arguments_get_documented_status_codes():
    code = CHILD.format(root=ROOT, seed=7, n=4000)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0, (r.returncode, r.stderr[-2000:])
    # every kind of outcome occurs: refusals, and calls that pass every host check and
    # stop at the first device query (no GPU here)
    for code in ("(1,", "(2,", "(4,"):
        assert code in r.stdout, r.stdout
