"""Per-role cycle counters of the packed-layout GEMMs (one CTA per tile and CTA pairs).

    python mixture_experts_softmax_b200/pipe_stats.py T MODE      # MODE: moe_set_cta_pairs mode 0..3

Builds an instrumented copy of the library (-DMOE_PIPE_STATS: every warp role of the GEMM kernels
adds up the cycles it spends waiting and working) under build/pipe_stats, runs the layer on T tokens
of the Grok-1 shape in the packed layout, and prints each role's mean cycles per CTA and launch.  A
development tool: the library itself is not instrumented."""
import ctypes, os, shutil, sys
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))   # the repository
SCR = os.path.join(ROOT, "build", "pipe_stats")
if not os.path.exists(os.path.join(SCR, "mixture_experts_softmax_b200", "libmoe_b200.so")):
    if os.path.exists(SCR):
        shutil.rmtree(SCR)
    os.makedirs(SCR)
    shutil.copytree(os.path.join(ROOT, "mixture_experts_softmax_b200"), os.path.join(SCR, "mixture_experts_softmax_b200"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "include"), os.path.join(SCR, "include"))
    sys.path.insert(0, SCR)
    import importlib.util
    spec = importlib.util.spec_from_file_location("b", os.path.join(SCR, "mixture_experts_softmax_b200", "build.py"))
    b = importlib.util.module_from_spec(spec); spec.loader.exec_module(b)
    b.build(force=True, extra=["-DMOE_PIPE_STATS"])
sys.path.insert(0, SCR)
sys.path.insert(1, ROOT)
import torch
import mixture_experts_softmax_b200 as moe
assert moe.LIB_PATH.startswith(SCR), moe.LIB_PATH
import moe_synth
lib = moe.lib()
T = int(sys.argv[1]); mode = int(sys.argv[2])
fns = {}
for nm in ("moe_debug_pipe_stats_ts", "moe_debug_pipe_stats_pair"):
    f = getattr(lib, nm); f.restype = ctypes.c_int; f.argtypes = [ctypes.c_void_p, ctypes.c_int]; fns[nm] = f
g = lib.moe_debug_pair_grid; g.restype = ctypes.c_int; g.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
inp = moe_synth.make_inputs("decode", device="cuda", T=T)
h = moe.MoELayer(6144, 32768)
moe.check(moe.moe_set_weight_layout(h.h, moe.MOE_LAYOUT_PACKED))
moe.check(moe.moe_set_cta_pairs(h.h, mode))
layer = moe.pack_layer(h.h, inp.layers[0])
out = torch.empty_like(inp.x)
for _ in range(3):
    moe.check(moe.moe_forward(h.h, T, inp.x, *moe.layer_args(layer), out))
torch.cuda.synchronize()
print("pair grids (up/down) bn=128:", g(1, 128, 148), g(0, 128, 148), " bn=32:", g(1, 32, 148), g(0, 32, 148))
bufs = {k: (ctypes.c_ulonglong * 64)() for k in fns}
for k, f in fns.items():
    f(bufs[k], 1)
N = 5 if T > 1000 else 50
e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
moe.check(moe.moe_set_profiling(h.h, True))
moe.moe_get_kernel_times(h.h)
for _ in range(N):
    moe.check(moe.moe_forward(h.h, T, inp.x, *moe.layer_args(layer), out))
torch.cuda.synchronize()
rc, kt = moe.moe_get_kernel_times(h.h)
print("ms per launch:", {k: round(v[0] / max(1, v[1]), 4) for k, v in kt.items() if v[1]})
for k, f in fns.items():
    f(bufs[k], 0)
names = ["total(thr0)", "tmaA wait stg_empty", "tmaB wait op_empty", "mma wait acc_empty", "mma wait a_full",
         "mma wait b_full", "mma issue", "epi wait acc_full", "epi work", "conv wait", "conv work", "conv st wait",
         "conv tail"]
per = {"tmaA": 1, "tmaB": 1, "mma": 2, "epi": 8, "conv": 8}
for k, buf in bufs.items():
    for kind, base in (("up", 0), ("down", 32)):
        for rank in ((0,) if k.endswith("_ts") else (0, 16)):
            tot = buf[base + rank]
            if tot == 0:
                continue
            ncta = 148 if k.endswith("_ts") else 74
            tot = tot / ncta / N
            print(f"== {k} {kind} rank{rank // 16}: mean cycles per CTA per launch {tot:.0f}")
            for i, nm in enumerate(names[1:], 1):
                role = nm.split()[0]
                div = per.get(role, 1)
                v = buf[base + rank + i] / ncta / N / div
                print(f"  {nm:22s} {v:10.0f}  {100 * v / tot:5.1f}%")
