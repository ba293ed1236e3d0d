"""Build libkdn.so in-tree with nvcc for sm_100a.

    python -m kalman_filter_linear_b200.build

The library is a plain shared object with a C ABI (include/kdn.h); it links
only the CUDA runtime.  Output: kalman_filter_linear_b200/libkdn.so.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, 'libkdn.so')
ARCH = ['-gencode', 'arch=compute_100a,code=sm_100a']


def nvcc():
    for cand in (os.environ.get('NVCC'), shutil.which('nvcc'), '/usr/local/cuda/bin/nvcc'):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError('nvcc not found')


def sources():
    return sorted(glob.glob(os.path.join(PKG, 'csrc', '*.cu')))


def build(verbose=False, extra=()):
    """Compile every source to an object in parallel, then link the library."""
    from concurrent.futures import ThreadPoolExecutor
    srcs = sources()
    objdir = os.path.join(ROOT, '_build')
    os.makedirs(objdir, exist_ok=True)
    flags = ['-Xcompiler', '-fPIC', '-O3', '-lineinfo', '-std=c++17', *ARCH,
             '-I', os.path.join(ROOT, 'include'), '--expt-relaxed-constexpr',
             '-Xptxas', '-warn-spills', *extra]

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + '.o')
        cmd = [nvcc(), '-c', *flags, '-o', obj, src]
        if verbose:
            print(' '.join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        return obj

    with ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, srcs))
    subprocess.run([nvcc(), '-shared', *ARCH, '-o', LIB + '.tmp', *objs, '-lcudart'], check=True)
    os.replace(LIB + '.tmp', LIB)
    return LIB


def is_stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(PKG, 'csrc', '*.cuh')) + \
        glob.glob(os.path.join(PKG, 'csrc', '*.h')) + glob.glob(os.path.join(ROOT, 'include', '*.h'))
    return any(os.path.getmtime(d) > t for d in deps)


if __name__ == '__main__':
    extra = sys.argv[1:]
    print(build(verbose=True, extra=extra))
