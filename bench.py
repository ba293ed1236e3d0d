#!/usr/bin/env python
"""Benchmark of the KDN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {kdn,reference}]

A step is one Isotropic KDN layer forward (kdn_iso_forward) over the whole
1.3B-layer-shaped workload: B=8, T=4096, H=16, d_k=d_v=128, bf16 q/k/v, fp32
decay / noise / state / output, inputs resident in HBM.  It covers the whole
hot path: per-token variance recursion, gains, chunkwise delta-rule engine,
outputs and final state.  Inputs (403 MB of q/k/v) are larger than the 126 MB
L2, so no flush is needed between steps.  Prints ONE JSON line (rank 0).

Also measured on the same run and reported under "secondary": the Diagonal
KDN forward at the same shape, the standalone variance scan (4096 x 65536),
the long-context diagonal forward (B1 T65536), the decode step (batch 256) and
the isotropic forward over 32768 tokens packed from sequences of mixed length
(kdn_forward_varlen), the dense (full-covariance) filter at d_k = d_v = 64
(kdn_exact_forward) and the information-form diagonal filter (kdn_kla_forward)
on the Diagonal KDN's inputs.

--impl reference times the fp64 CPU oracle (the correctness reference) on a
bounded sample of the same workload on the host cores.

Multi-GPU (torchrun, one process per GPU): every rank runs its own copy of
the workload; (b, h) heads are independent, so there is no collective on the
data path ("weak" scaling).  Time is the max over ranks of each rank's
CUDA-event time.
"""
from __future__ import annotations

import argparse
import itertools
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = 'KDN layer fwd tokens/s (B8 T4096 H16 d128)'
WORKLOAD = 'iso_1p3b'


def peaks():
    path = os.path.join(ROOT, 'MEASURED_PEAKS.json')
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p['hbm_gbs']), float(p['bf16_tflops']), 'measured'
    return 6650.0, 1590.0, 'fallback'


def layer_bytes(variant, B, T, H, dk, dv, in_bytes=2):
    """Algorithmic HBM bytes of one layer forward: read q, k, v, a, w, r;
    write o (fp32), S_T, p_T (S0 = 0 and p0 = 1 are not read)."""
    qkv = B * T * H * (2 * dk + dv) * in_bytes
    ar = 2 * B * T * H * 4
    w = B * T * H * (dk if variant == 'diag' else 1) * 4
    o = B * T * H * dv * 4
    st = B * H * dv * dk * 4 + B * H * (dk if variant == 'diag' else 1) * 4
    return qkv + ar + w + o + st


PROFILE = os.path.join(ROOT, 'profiles', 'chunk_engine_ws_iso_B4_T4096_H16_d128.md')
ENGINE_SOURCES = [os.path.join(ROOT, 'kalman_filter_linear_b200', 'csrc', f)
                  for f in ('chunk_engine.cu', 'kdn_common.cuh')]


def captured_traffic(heads):
    """DRAM bytes (read + write) of one launch over `heads` heads, scaled from
    the committed ncu capture of the isotropic engine -- or None when the
    engine's sources changed since that capture (its counters no longer
    describe the kernel that runs)."""
    import hashlib
    try:
        text = open(PROFILE).read()
        per_head = float(re.search(r'^traffic-bytes-per-head: (\d+)', text, re.M).group(1))
        digest = re.search(r'^source-sha256-16: ([0-9a-f]+)', text, re.M).group(1)
    except (OSError, AttributeError):
        return None
    h = hashlib.sha256()
    for f in ENGINE_SOURCES:
        h.update(open(f, 'rb').read())
    return per_head * heads if h.hexdigest()[:16] == digest else None


def decode_bytes(B, H, dk, dv):
    """Per decode step (diagonal): S read+write, p read+write, q/k/v bf16,
    a/r, per-dimension w, o fp32."""
    return (2 * B * H * dv * dk * 4 + 2 * B * H * dk * 4 + B * H * (2 * dk + dv) * 2 +
            2 * B * H * 4 + B * H * dk * 4 + B * H * dv * 4)


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""
    FIELDS = ('clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,'
              'clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,'
              'clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap')

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def _once(self):
        try:
            out = subprocess.run(['nvidia-smi', '-i', str(self.gpu), '--query-gpu=' + self.FIELDS,
                                  '--format=csv,noheader,nounits'], capture_output=True,
                                 text=True, timeout=10)
            return out.stdout.strip().splitlines()
        except Exception:
            return []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ['nvidia-smi', '-i', str(self.gpu), '--query-gpu=' + self.FIELDS,
                 '--format=csv,noheader,nounits', '-lms', '100'],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        if not self.lines:
            self.lines = self._once()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ['hw_slowdown', 'hw_thermal_slowdown', 'sw_thermal_slowdown', 'sw_power_cap']
        for line in self.lines:
            f = [x.strip() for x in line.split(',')]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                smax = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == 'active':
                    reasons.add(n)
        if not sm:
            return {'sm_mhz': None, 'sm_max_mhz': None, 'reasons': ['unavailable'], 'samples': 0}
        return {'sm_mhz': statistics.median(sm), 'sm_max_mhz': smax, 'reasons': sorted(reasons),
                'samples': len(sm)}


def max_over_ranks(value, dist, device):
    """The largest of every rank's value (all-reduce MAX); the value itself
    when there is one rank."""
    import torch
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms_max_per_step):
    """Units per second of the whole job: every rank processes
    `units_per_rank` per step, and a step lasts as long as the slowest rank."""
    return world * units_per_rank / (ms_max_per_step / 1000.0)


def time_launches(fn, steps, warmup, stream):
    """CUDA-event time (ms) of `steps` back-to-back calls of fn on `stream`."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


# ---------------------------------------------------------------- reference
# The fp64 oracle, as it stands, on the host cores.  Heads (b, h) are
# independent, so a pool of processes (spawned, never forked after CUDA use)
# runs the oracle's token loop over disjoint sets of heads, one BLAS/OpenMP
# thread each; the parent times the whole pool on the wall clock.
_ORACLE_X = None


def _oracle_init(spec):
    """Worker start: attach the shared input arrays (no copy)."""
    global _ORACLE_X
    import numpy as np
    from multiprocessing import shared_memory
    _ORACLE_X = {}
    for n, (name, shape) in spec.items():
        shm = shared_memory.SharedMemory(name=name)
        _ORACLE_X[n] = (shm, np.ndarray(shape, dtype=np.float32, buffer=shm.buf))


def _oracle_heads(job):
    """Worker: the isotropic oracle over heads [h0, h1) (each head a batch
    entry of its own) for tokens [t0, t1); returns the elapsed seconds."""
    h0, h1, t0, t1 = job
    from oracle import kdn_ref
    xs = [_ORACLE_X[n][1][h0:h1, t0:t1] for n in 'qkvawr']
    S0, p0 = _ORACLE_STATE.get((h0, h1), (None, None)) if t0 > 0 else (None, None)
    t = time.perf_counter()
    _, S, p = kdn_ref.iso_forward(*xs, S0=S0, p0=p0)
    el = time.perf_counter() - t
    _ORACLE_STATE[(h0, h1)] = (S, p)  # the next window continues from here
    return el


_ORACLE_STATE = {}


class OraclePool:
    """A spawn pool over the sample's inputs, held once in shared memory as
    fp32 [B*H, T, 1, d] (heads as batch entries; the bf16 values are exact in
    fp32, and the oracle converts to fp64 itself); run(t0, t1) covers every
    head for tokens [t0, t1)."""

    def __init__(self, B, T, H, d, seed, dtype):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        import numpy as np
        from kalman_filter_linear_b200 import synth
        x = synth.layer_inputs(B, T, H, d, d, 'iso', seed, dtype)
        heads = B * H
        self.shms, spec = [], {}
        for n in 'qkvawr':
            t = x[n].float().numpy()
            t = t.transpose(0, 2, 1, *range(3, t.ndim)).reshape(heads, T, *t.shape[3:])
            t = t[:, :, None]
            shm = shared_memory.SharedMemory(create=True, size=max(t.nbytes, 1))
            np.ndarray(t.shape, dtype=np.float32, buffer=shm.buf)[...] = t
            self.shms.append(shm)
            spec[n] = (shm.name, t.shape)
        del x
        try:
            cpus = len(os.sched_getaffinity(0))
        except AttributeError:
            cpus = os.cpu_count() or 1
        self.cpus = cpus
        self.procs = max(1, min(cpus, heads))
        self.B, self.heads = B, heads
        bounds = [heads * i // self.procs for i in range(self.procs + 1)]
        self.groups = [(bounds[i], bounds[i + 1]) for i in range(self.procs)]
        env = {k: os.environ.get(k) for k in ('OMP_NUM_THREADS', 'OPENBLAS_NUM_THREADS',
                                              'MKL_NUM_THREADS')}
        for k in env:
            os.environ[k] = '1'
        try:
            self.pool = mp.get_context('spawn').Pool(self.procs, initializer=_oracle_init,
                                                     initargs=(spec,))
        finally:
            for k, v in env.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.run(0, 1)  # every worker has imported the oracle

    def run(self, t0, t1):
        t = time.perf_counter()
        self.pool.map(_oracle_heads, [(h0, h1, t0, t1) for h0, h1 in self.groups],
                      chunksize=1)
        return time.perf_counter() - t

    def describe(self):
        return {'cores': self.procs,
                'threads': f'{self.procs} processes x 1 BLAS/OpenMP thread '
                           f'({self.cpus} host CPUs available)'}

    def close(self):
        self.pool.close()
        self.pool.join()
        for shm in self.shms:
            shm.close()
            shm.unlink()


def run_reference(args, rank):
    """The fp64 CPU oracle on a bounded sample of the workload, on all the
    host cores (rank 0 only; other ranks exit without work)."""
    if rank != 0:
        return
    from kalman_filter_linear_b200 import synth
    cfg = synth.WORKLOADS[WORKLOAD]
    B, T, H, d = cfg['B'], cfg['T'], cfg['H'], cfg['dk']
    # tokens of all B*H heads per step, a bounded sample of the workload: 64
    # at up to 50 steps, fewer for more steps, so the run stays within minutes
    tok = max(1, min(64, (64 * 50) // max(args.steps, 1)))
    pool = OraclePool(B, tok, H, d, cfg['seed'], cfg['dtype'])
    for _ in range(args.warmup):
        pool.run(0, tok)
    el = sum(pool.run(0, tok) for _ in range(args.steps))
    pool.close()
    value = B * tok * args.steps / el
    desc = pool.describe()
    print(json.dumps({
        'impl': 'reference', 'metric': METRIC, 'value': value, 'unit': 'tokens/s',
        'n_gpus': args.gpus, 'steps': args.steps, 'warmup': args.warmup,
        'ms_per_step': 1000 * el / args.steps, 'higher_is_better': True, 'scaling': 'weak',
        'vs_baseline': None, 'dtype': 'f64', 'data': 'synthetic',
        'config': {'workload': WORKLOAD, 'B': B, 'T': T, 'H': H, 'dk': d, 'dv': d,
                   'sample': f'first {tok} tokens of all {B}x{H} heads per step'},
        'cpu_baseline': {'value': value, 'unit': 'tokens/s', 'cores': desc['cores'],
                         'threads': desc['threads'], 'kind': 'oracle',
                         'sample': f'{tok} tokens x {B * H} heads per step, fp64 NumPy '
                                   'token loop, heads split over the processes'},
        'e2e': {'value': value, 'unit': 'tokens/s', 'h2d_bytes_per_step': 0,
                'd2h_bytes_per_step': 0}}))


def cpu_baseline(seconds=12.0):
    """Time the oracle as it stands on a bounded sample of the workload (all
    B*H heads, a run of tokens sized to about `seconds` of wall time) on all
    the host cores."""
    from kalman_filter_linear_b200 import synth
    cfg = synth.WORKLOADS[WORKLOAD]
    B, H, d = cfg['B'], cfg['H'], cfg['dk']
    span, window = cfg['T'], 32
    pool = OraclePool(B, span, H, d, cfg['seed'], cfg['dtype'])
    # consecutive windows from the first token on, each continuing from the
    # state the previous one left, until `seconds` have passed or the
    # sequence ends
    tok, el = 0, 0.0
    while tok < span and el < seconds:
        el += pool.run(tok, min(tok + window, span))
        tok = min(tok + window, span)
    pool.close()
    desc = pool.describe()
    return {'value': B * tok / el, 'unit': 'tokens/s', 'cores': desc['cores'],
            'threads': desc['threads'], 'kind': 'oracle',
            'sample': f'tokens [0, {tok}) of all {B}x{H} heads (B8 H16 d128), fp64 NumPy '
                      f'token loop, heads split over {desc["cores"]} processes, '
                      f'{el:.1f} s wall'}


# --------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument('--gpus', type=int, default=1)
    ap.add_argument('--steps', type=int, default=2000)
    ap.add_argument('--warmup', type=int, default=5)
    ap.add_argument('--impl', default='kdn', choices=['kdn', 'reference'])
    ap.add_argument('--no-secondary', action='store_true')
    ap.add_argument('--no-cpu-baseline', action='store_true')
    ap.add_argument('--only', choices=['iso', 'diag', 'scan', 'decode', 'varlen', 'exact', 'kla',
                                       'bwd', 'bwd128'],
                    help='run only this kernel (for profiler captures) and print its timing')
    ap.add_argument('--B', type=int, default=None, help='batch override for --only')
    ap.add_argument('--T', type=int, default=None, help='length override for --only')
    args = ap.parse_args()
    if args.only:
        run_only(args)
        return
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get('RANK', '0'))
    world = int(os.environ.get('WORLD_SIZE', '1'))
    local = int(os.environ.get('LOCAL_RANK', '0'))
    if args.impl == 'reference':
        run_reference(args, rank)
        return

    import torch
    from kalman_filter_linear_b200 import kdn, synth

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group('nccl', timeout=datetime.timedelta(seconds=120))
    dev = torch.device('cuda', local)
    stream = torch.cuda.current_stream()
    hbm_peak, tf_peak, peak_kind = peaks()

    cfg = synth.WORKLOADS[WORKLOAD]
    B, T, H, d = cfg['B'], cfg['T'], cfg['H'], cfg['dk']
    host = synth.layer_inputs(B, T, H, d, d, 'iso', cfg['seed'] + 1000 * rank, cfg['dtype'])
    x = {k: v.to(dev) for k, v in host.items()}
    ws = torch.empty(max(kdn.kdn_forward_workspace_size(kdn.KDN_ISO, B, T, H, d, d), 256),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((B, T, H, d), dtype=torch.float32, device=dev)
    S_out = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    p_out = torch.empty((B, H), dtype=torch.float32, device=dev)

    def step():
        kdn.kdn_iso_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], o=o, S_out=S_out,
                            p_out=p_out, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = time_launches(step, args.steps, 0, stream)
    if dist:
        dist.barrier()
    ms_max = max_over_ranks(ms, dist, dev)
    ms_step = ms_max / args.steps
    value = whole_job_rate(B * T, world, ms_step)
    alg = layer_bytes('iso', B, T, H, d, d)
    achieved = alg / (ms / args.steps / 1000.0) / 1e9

    # ---- end to end through the public API: pinned host in, result out.
    # kdn_forward_host copies each batch entry in, runs it and copies it back
    # on two alternating streams, so the copies in and out overlap.
    pinned = {k: v.pin_memory() for k, v in host.items()}
    o_host = torch.empty((B, T, H, d), dtype=torch.float32).pin_memory()
    S_host = torch.empty((B, H, d, d), dtype=torch.float32).pin_memory()
    p_host = torch.empty((B, H), dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = o_host.numel() * 4 + S_host.numel() * 4 + p_host.numel() * 4
    ws_host = torch.empty(kdn.kdn_forward_host_workspace_size(kdn.KDN_ISO, B, T, H, d, d,
                                                              kdn.KDN_BF16, kdn.KDN_CHUNK_AUTO, 1),
                          dtype=torch.uint8, device=dev)

    def e2e_step():
        kdn.kdn_forward_host(kdn.KDN_ISO, pinned['q'], pinned['k'], pinned['v'], pinned['a'],
                             pinned['w'], pinned['r'], slice_b=1, o=o_host, S_out=S_host,
                             p_out=p_host, workspace=ws_host, device=dev)

    e2e_steps = max(3, min(args.steps, 10))
    ms_e2e = time_launches(e2e_step, e2e_steps, 2, stream) / e2e_steps
    e2e_value = whole_job_rate(B * T, world, max_over_ranks(ms_e2e, dist, dev))

    # secondary lines at N = 1 only: at N > 1 the other ranks would wait at the
    # closing barrier (under the process group's timeout) while rank 0 measures
    secondary = {}
    if not args.no_secondary and rank == 0 and world == 1:
        secondary = measure_secondary(kdn, synth, dev, stream, hbm_peak, tf_peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        'metric': METRIC, 'value': value, 'unit': 'tokens/s', 'n_gpus': world,
        'steps': args.steps, 'warmup': args.warmup, 'ms_per_step': ms_step,
        'higher_is_better': True, 'scaling': 'weak', 'vs_baseline': None, 'dtype': 'bf16',
        'data': 'synthetic',
        'config': {'workload': WORKLOAD, 'B': B, 'T': T, 'H': H, 'dk': d, 'dv': d,
                   'chunk': 64, 'inputs': 'q/k/v bf16, a/w/r fp32, S0=0, p0=1',
                   'outputs': 'o fp32 [B,T,H,dv], S_T fp32, p_T fp32',
                   'arithmetic': 'bf16 hi/lo tensor-core operands, fp32 accumulate, '
                                 'state and variance',
                   'l2': 'inputs (403 MB q/k/v) larger than the 126 MB L2; no flush',
                   'parallelism': f'dp{world} (independent replicas, no collective)'},
        'roofline': {'bound': 'hbm', 'achieved': achieved, 'peak': hbm_peak, 'unit': 'GB/s',
                     'frac': achieved / hbm_peak, 'traffic': captured_traffic(B * H),
                     'algorithmic_bytes': alg, 'peak_source': peak_kind},
        'e2e': {'value': e2e_value, 'unit': 'tokens/s', 'h2d_bytes_per_step': h2d,
                'd2h_bytes_per_step': d2h},
        'gpu_launches': args.steps,
        'clocks': clk.summary(),
        'cpu_baseline': cpu,
        'secondary': secondary,
    }
    print(json.dumps(line))


def run_only(args):
    """One kernel on its own, for profiler captures: `steps` timed launches
    after `warmup` untimed ones."""
    import torch
    from kalman_filter_linear_b200 import kdn, synth
    dev = torch.device('cuda', 0)
    stream = torch.cuda.current_stream()
    if args.only in ('iso', 'diag'):
        c = synth.WORKLOADS['iso_1p3b' if args.only == 'iso' else 'diag_1p3b']
        B = args.B or c['B']
        T = args.T or c['T']
        H, d = c['H'], c['dk']
        x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, d, d, args.only, c['seed'],
                                                         c['dtype']).items()}
        var = kdn.KDN_ISO if args.only == 'iso' else kdn.KDN_DIAG
        ws = torch.empty(max(kdn.kdn_forward_workspace_size(var, B, T, H, d, d), 256),
                         dtype=torch.uint8, device=dev)
        fwd = kdn.kdn_iso_forward if args.only == 'iso' else kdn.kdn_diag_forward
        f = lambda: fwd(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], workspace=ws)
        units, alg = B * T, layer_bytes(args.only, B, T, H, d, d)
    elif args.only == 'scan':
        c = synth.WORKLOADS['scan']
        N = args.B or c['N']
        T = args.T or c['T']
        xs = {k: v.to(dev) for k, v in synth.scan_inputs(N, T, c['seed']).items()}
        lam = torch.empty_like(xs['a'])
        wss = torch.empty(kdn.kdn_mobius_scan_workspace_size(N, T), dtype=torch.uint8,
                          device=dev)
        f = lambda: kdn.kdn_mobius_scan(xs['a'], xs['w'], xs['r'], xs['n'], None,
                                        c['info_scale'], lambda_out=lam, workspace=wss)
        units, alg = N * T, N * T * 20
    elif args.only == 'varlen':
        f, units, alg, _ = varlen_case(kdn, synth, dev)
    elif args.only == 'exact':
        f, units, alg, _ = exact_case(kdn, synth, dev, args.B, args.T)
    elif args.only == 'bwd':
        c = synth.WORKLOADS['exact_d64']
        B, T, H, d = args.B or c['B'], args.T or c['T'], c['H'], c['dk']
        x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, d, d, 'iso', c['seed'],
                                                         c['dtype']).items()}
        dO = torch.randn((B, T, H, d),
                         generator=torch.Generator().manual_seed(c['seed'] + 100)).to(dev)
        wsb = torch.empty(kdn.kdn_backward_workspace_size(kdn.KDN_ISO, B, T, H, d, d),
                          dtype=torch.uint8, device=dev)
        f = lambda: kdn.kdn_backward('iso', x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], dO,
                                     workspace=wsb)
        units, alg = B * T, backward_bytes(B, T, H, d)
    elif args.only == 'bwd128':
        f, units, alg, _ = backward128_case(kdn, synth, dev, args.B, args.T)
    elif args.only == 'kla':
        c = synth.WORKLOADS['diag_1p3b']
        B, T, H, d = args.B or c['B'], args.T or c['T'], c['H'], c['dk']
        x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, d, d, 'diag', c['seed'],
                                                         c['dtype']).items()}
        f = lambda: kdn.kdn_kla_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'])
        units, alg = B * T, layer_bytes('diag', B, T, H, d, d)
    else:
        c = synth.WORKLOADS['diag_long']
        B = args.B or c['decode_batch']
        H, d = c['H'], c['dk']
        st = synth.decode_state(B, H, d, d, 'diag', seed=c['seed'])
        Sd, pd = st['S'].to(dev), st['p'].to(dev)
        xd = {k: v.to(dev) for k, v in synth.decode_inputs(B, H, d, d, 'diag', c['seed']).items()}
        od = torch.empty((B, H, d), dtype=torch.float32, device=dev)
        f = lambda: kdn.kdn_decode_step('diag', xd['q'], xd['k'], xd['v'], xd['a'], xd['w'],
                                        xd['r'], Sd, pd, o=od)
        units, alg = B, decode_bytes(B, H, d, d)
    ms = time_launches(f, args.steps, args.warmup, stream) / max(args.steps, 1)
    print(json.dumps({'only': args.only, 'ms': ms, 'units_per_s': units / ms * 1e3,
                      'achieved_gbs': alg / ms / 1e6, 'algorithmic_bytes': alg}))


def varlen_case(kdn, synth, dev):
    """The packed isotropic forward: (launch fn, tokens, algorithmic bytes,
    description)."""
    import torch
    c = synth.WORKLOADS['iso_varlen']
    lengths = synth.packed_lengths(c['total'], c['seed'], c['min_len'], c['max_len'])
    total, H, d, N = c['total'], c['H'], c['dk'], len(lengths)
    x = synth.layer_inputs(1, total, H, d, d, 'iso', c['seed'], c['dtype'])
    x = {k: v[0].to(dev) for k, v in x.items()}
    cu = torch.tensor([0] + list(itertools.accumulate(lengths)),
                      dtype=torch.int32, device=dev)
    ws = torch.empty(kdn.kdn_forward_varlen_workspace_size(kdn.KDN_ISO, N, H, d, d),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((total, H, d), dtype=torch.float32, device=dev)
    S = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    p = torch.empty((N, H), dtype=torch.float32, device=dev)
    f = lambda: kdn.kdn_forward_varlen(kdn.KDN_ISO, x['q'], x['k'], x['v'], x['a'], x['w'],
                                       x['r'], cu, o=o, S_out=S, p_out=p, workspace=ws)
    # tokens move as in one B1 T=total launch; the final state is per sequence
    alg = layer_bytes('iso', 1, total, H, d, d) + (N - 1) * H * (d * d + 1) * 4
    desc = {'sequences': N, 'tokens': total, 'max_len': max(lengths),
            'min_len': min(lengths), 'H': H, 'd': d}
    return f, total, alg, desc


def backward_bytes(B, T, H, d, variant='iso', in_bytes=2, ck=16):
    """Algorithmic HBM bytes of one backward call at d_k = d_v = d: inputs
    read twice (the forward again, then the backward), dO read, the forward's
    o written, the state checkpoints (every ck-th token) and the variance of
    every token written and read once, the gradients written.  The rebuilt
    states of each 16-token block stay in a per-CTA scratch that L2 holds."""
    dim = d if variant == 'diag' else 1
    inp = B * T * H * (3 * d * in_bytes + (2 + dim) * 4)
    ck_states = B * H * (-(-T // ck)) * d * d * 4
    grads = B * T * H * (3 * d + 2 + dim) * 4
    return (2 * inp + 2 * B * T * H * d * 4 + 2 * ck_states + 2 * B * H * T * dim * 4 + grads)


def backward128_case(kdn, synth, dev, B=None, T=None, variant='iso'):
    """The backward pass at the 1.3B-layer shape (d_k = d_v = 128): (launch
    fn, tokens, algorithmic bytes, description)."""
    import torch
    c = synth.WORKLOADS['iso_1p3b' if variant == 'iso' else 'diag_1p3b']
    B, T, H, d = B or c['B'], T or c['T'], c['H'], c['dk']
    x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, d, d, variant, c['seed'],
                                                     c['dtype']).items()}
    dO = torch.randn((B, T, H, d), generator=torch.Generator().manual_seed(c['seed'] + 100)).to(dev)
    var = kdn.KDN_ISO if variant == 'iso' else kdn.KDN_DIAG
    wsb = torch.empty(kdn.kdn_backward_workspace_size(var, B, T, H, d, d), dtype=torch.uint8,
                      device=dev)
    f = lambda: kdn.kdn_backward(variant, x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], dO,
                                 workspace=wsb)
    return f, B * T, backward_bytes(B, T, H, d, variant), {'B': B, 'T': T, 'H': H, 'd': d,
                                                             'variant': variant}


def exact_bytes(B, T, H, dk, dv, in_bytes=2):
    """Algorithmic HBM bytes of the dense filter (W = w I): read q, k, v, a,
    w, r; write o (fp32), S_T and P_T."""
    return (B * T * H * ((2 * dk + dv) * in_bytes + 3 * 4 + dv * 4) +
            B * H * (dv * dk + dk * dk) * 4)


def exact_flops(B, T, H, dk, dv):
    """Algorithmic FLOPs of the dense filter (an FMA counts 2): per token and
    head, P- = a^2 P + W (2 dk^2), u = P- k (2 dk^2), P = P- - u u^T / s
    (3 dk^2); S k and S q (4 dv dk), S = a S + e g^T (3 dv dk)."""
    return B * T * H * (7 * dk * dk + 7 * dv * dk)


# FP32 peak of the CUDA cores (no tensor cores): 148 SMs x 128 FP32 lanes x
# 2 FLOPs per FMA x 1.965 GHz (the B200's maximum SM clock)
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def kla_engine_flops(B, T, H):
    """Tensor FLOPs the KLA engine executes (bf16 hi/lo terms included): per
    64-token chunk and head, MMA-A 16 and MMA-O 24 instructions of 128x64x16,
    MMA-I 12 of 128x64x16, MMA-dS 8 of 128x128x16."""
    per_chunk = (16 + 24 + 12) * 2 * 128 * 64 * 16 + 8 * 2 * 128 * 128 * 16
    return B * H * ((T + 63) // 64) * per_chunk


def exact_case(kdn, synth, dev, B=None, T=None):
    """The dense filter: (launch fn, tokens, algorithmic bytes, description)."""
    import torch
    c = synth.WORKLOADS['exact_d64']
    B, T = B or c['B'], T or c['T']
    H, dk, dv = c['H'], c['dk'], c['dv']
    x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, dk, dv, c['variant'], c['seed'],
                                                     c['dtype']).items()}
    o = torch.empty((B, T, H, dv), dtype=torch.float32, device=dev)
    S = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    P = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    f = lambda: kdn.kdn_exact_forward(c['variant'], x['q'], x['k'], x['v'], x['a'], x['w'],
                                      x['r'], o=o, S_out=S, P_out=P)
    return f, B * T, exact_bytes(B, T, H, dk, dv), {'B': B, 'T': T, 'H': H, 'dk': dk, 'dv': dv}


def measure_secondary(kdn, synth, dev, stream, hbm_peak, tensor_peak):
    import torch
    out = {}
    # diagonal forward, same shape
    c = synth.WORKLOADS['diag_1p3b']
    B, T, H, d = c['B'], c['T'], c['H'], c['dk']
    x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, d, d, 'diag', c['seed'],
                                                     c['dtype']).items()}
    ws = torch.empty(max(kdn.kdn_forward_workspace_size(kdn.KDN_DIAG, B, T, H, d, d), 256),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((B, T, H, d), dtype=torch.float32, device=dev)
    S = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    p = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    f = lambda: kdn.kdn_diag_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], o=o,
                                     S_out=S, p_out=p, workspace=ws)
    n = 10
    ms = time_launches(f, n, 3, stream) / n
    alg = layer_bytes('diag', B, T, H, d, d)
    out['diag_1p3b'] = {'tokens_per_s': B * T / ms * 1e3, 'ms': ms,
                        'achieved_gbs': alg / ms / 1e6, 'frac': alg / ms / 1e6 / hbm_peak,
                        'algorithmic_bytes': alg}
    del x, o, S, p
    # long-context diagonal forward, B1 T65536 H16
    c = synth.WORKLOADS['diag_long']
    B, T, H, d = c['B'], c['T'], c['H'], c['dk']
    x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, d, d, 'diag', c['seed'],
                                                     c['dtype']).items()}
    ws = torch.empty(max(kdn.kdn_forward_workspace_size(kdn.KDN_DIAG, B, T, H, d, d), 256),
                     dtype=torch.uint8, device=dev)
    f = lambda: kdn.kdn_diag_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'],
                                     workspace=ws)
    ms = time_launches(f, 3, 2, stream) / 3
    alg = layer_bytes('diag', B, T, H, d, d)
    out['diag_long'] = {'tokens_per_s': B * T / ms * 1e3, 'ms': ms,
                        'achieved_gbs': alg / ms / 1e6, 'frac': alg / ms / 1e6 / hbm_peak,
                        'algorithmic_bytes': alg}
    del x, ws
    # standalone variance scan
    c = synth.WORKLOADS['scan']
    N, Tn = c['N'], c['T']
    xs = {k: v.to(dev) for k, v in synth.scan_inputs(N, Tn, c['seed']).items()}
    lam = torch.empty_like(xs['a'])
    wss = torch.empty(kdn.kdn_mobius_scan_workspace_size(N, Tn), dtype=torch.uint8, device=dev)
    f = lambda: kdn.kdn_mobius_scan(xs['a'], xs['w'], xs['r'], xs['n'], None, c['info_scale'],
                                    lambda_out=lam, workspace=wss)
    ms = time_launches(f, n, 3, stream) / n
    alg = N * Tn * 20
    out['scan'] = {'steps_per_s': N * Tn / ms * 1e3, 'ms': ms, 'achieved_gbs': alg / ms / 1e6,
                   'frac': alg / ms / 1e6 / hbm_peak, 'algorithmic_bytes': alg}
    del xs, lam, wss
    # decode step, batch 256, diagonal
    c = synth.WORKLOADS['diag_long']
    Bd, H, d = c['decode_batch'], c['H'], c['dk']
    st = synth.decode_state(Bd, H, d, d, 'diag', seed=c['seed'])
    Sd, pd = st['S'].to(dev), st['p'].to(dev)
    xd = {k: v.to(dev) for k, v in synth.decode_inputs(Bd, H, d, d, 'diag', c['seed']).items()}
    od = torch.empty((Bd, H, d), dtype=torch.float32, device=dev)
    f = lambda: kdn.kdn_decode_step('diag', xd['q'], xd['k'], xd['v'], xd['a'], xd['w'], xd['r'],
                                    Sd, pd, o=od)
    n = 50
    ms = time_launches(f, n, 5, stream) / n
    alg = decode_bytes(Bd, H, d, d)
    out['decode'] = {'tokens_per_s': Bd / ms * 1e3, 'ms': ms, 'achieved_gbs': alg / ms / 1e6,
                     'frac': alg / ms / 1e6 / hbm_peak, 'algorithmic_bytes': alg}
    del Sd, pd, xd, od
    # packed variable-length isotropic forward, 32768 tokens
    f, units, alg, desc = varlen_case(kdn, synth, dev)
    n = 10
    ms = time_launches(f, n, 3, stream) / n
    out['iso_varlen'] = {'tokens_per_s': units / ms * 1e3, 'ms': ms,
                         'achieved_gbs': alg / ms / 1e6, 'frac': alg / ms / 1e6 / hbm_peak,
                         'algorithmic_bytes': alg, **desc}
    # information-form diagonal filter (KLA) on the Diagonal KDN's inputs: the
    # chunked tensor-core engine (kdn_kla_forward_ws), and the token-recurrent
    # kernel (kdn_kla_forward) for comparison
    c = synth.WORKLOADS['diag_1p3b']
    B, T, H, d = c['B'], c['T'], c['H'], c['dk']
    x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, d, d, 'diag', c['seed'],
                                                     c['dtype']).items()}
    o = torch.empty((B, T, H, d), dtype=torch.float32, device=dev)
    S = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    lam = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    wsk = torch.zeros(kdn.kdn_kla_workspace_size(B, T, H, d, d), dtype=torch.uint8, device=dev)
    f = lambda: kdn.kdn_kla_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], o=o,
                                    S_out=S, lam_out=lam, workspace=wsk)
    n = 10
    ms = time_launches(f, n, 3, stream) / n
    alg = layer_bytes('diag', B, T, H, d, d)
    tfl = kla_engine_flops(B, T, H)
    out['kla_1p3b'] = {'tokens_per_s': B * T / ms * 1e3, 'ms': ms, 'achieved_gbs': alg / ms / 1e6,
                       'frac': alg / ms / 1e6 / hbm_peak, 'algorithmic_bytes': alg,
                       'tensor': {'executed_flops': tfl, 'achieved_tflops': tfl / ms / 1e9,
                                  'peak_tflops': tensor_peak,
                                  'frac': tfl / ms / 1e9 / tensor_peak}}
    fr = lambda: kdn.kdn_kla_forward(x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], o=o,
                                     S_out=S, lam_out=lam, recurrent=True)
    n = 5
    ms = time_launches(fr, n, 3, stream) / n
    fl = B * T * H * 5 * d * d  # S f + v u^T (3 per element), S q (2)
    out['kla_recurrent_1p3b'] = {
        'tokens_per_s': B * T / ms * 1e3, 'ms': ms, 'achieved_gbs': alg / ms / 1e6,
        'frac': alg / ms / 1e6 / hbm_peak, 'algorithmic_bytes': alg,
        'alu': {'achieved_tflops': fl / ms / 1e9, 'peak_tflops': FP32_PEAK_TFLOPS,
                'frac': fl / ms / 1e9 / FP32_PEAK_TFLOPS, 'flops': fl}}
    del x, o, S, lam
    # backward pass (token-recurrent), B8 T4096 H16 d64, isotropic
    c = synth.WORKLOADS['exact_d64']
    B, T, H, d = c['B'], c['T'], c['H'], c['dk']
    x = {k: v.to(dev) for k, v in synth.layer_inputs(B, T, H, d, d, 'iso', c['seed'],
                                                     c['dtype']).items()}
    dO = torch.randn((B, T, H, d),
                     generator=torch.Generator().manual_seed(c['seed'] + 100)).to(dev)
    wsb = torch.empty(kdn.kdn_backward_workspace_size(kdn.KDN_ISO, B, T, H, d, d),
                      dtype=torch.uint8, device=dev)
    f = lambda: kdn.kdn_backward('iso', x['q'], x['k'], x['v'], x['a'], x['w'], x['r'], dO,
                                 workspace=wsb)
    n = 2
    ms = time_launches(f, n, 2, stream) / n
    alg = backward_bytes(B, T, H, d)
    out['backward_d64'] = {'tokens_per_s': B * T / ms * 1e3, 'ms': ms,
                           'achieved_gbs': alg / ms / 1e6, 'frac': alg / ms / 1e6 / hbm_peak,
                           'algorithmic_bytes': alg, 'B': B, 'T': T, 'H': H, 'd': d}
    del x, dO, wsb
    # backward pass at the 1.3B-layer shape, B8 T4096 H16 d128, isotropic
    f, units, alg, desc = backward128_case(kdn, synth, dev)
    n = 2
    ms = time_launches(f, n, 2, stream) / n
    out['backward_d128'] = {'tokens_per_s': units / ms * 1e3, 'ms': ms,
                            'achieved_gbs': alg / ms / 1e6, 'frac': alg / ms / 1e6 / hbm_peak,
                            'algorithmic_bytes': alg, **desc}
    del f
    torch.cuda.empty_cache()
    # dense (full-covariance) filter, B8 T4096 H16 d64
    f, units, alg, desc = exact_case(kdn, synth, dev)
    n = 3
    ms = time_launches(f, n, 3, stream) / n
    fl = exact_flops(desc['B'], desc['T'], desc['H'], desc['dk'], desc['dv'])
    out['exact_d64'] = {'tokens_per_s': units / ms * 1e3, 'ms': ms,
                        'achieved_gbs': alg / ms / 1e6, 'frac': alg / ms / 1e6 / hbm_peak,
                        'algorithmic_bytes': alg,
                        'alu': {'achieved_tflops': fl / ms / 1e9, 'peak_tflops': FP32_PEAK_TFLOPS,
                                'frac': fl / ms / 1e9 / FP32_PEAK_TFLOPS, 'flops': fl},
                        **desc}
    return out


if __name__ == '__main__':
    main()
