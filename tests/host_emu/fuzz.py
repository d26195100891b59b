"""Randomised shapes through the host-emulated kernels (SIMT chunk forward and
backward with the gate variants, decode step, tensor-core chunk kernel with
chunk states / per-head gate / transition, segment combine, layer prologue
and epilogue) against the FP64 oracle.

TEST INFRASTRUCTURE, run by hand (not by pytest), with the AddressSanitizer
runtime preloaded after emu_build.py has built the library:
    LD_PRELOAD=$(g++ -print-file-name=libasan.so) ASAN_OPTIONS=detect_leaks=0 \
        python tests/host_emu/fuzz.py SEED SECONDS
Prints MISMATCH / ERROR lines and a final count."""
import ctypes
import os
import random
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import run_parity as R  # noqa: E402

lib = ctypes.CDLL(os.path.join(HERE, "_build", "libkda_host_emu.so"))
lib.emu_compose.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 4
rng = random.Random(int(sys.argv[1]) if len(sys.argv) > 1 else 0)
t_end = time.time() + float(sys.argv[2] if len(sys.argv) > 2 else 600)
n = bad = 0
while time.time() < t_end:
    kind = rng.choice(["simt", "simt", "step", "tc", "compose", "layer"])
    try:
        if kind == "simt":
            H = rng.choice([1, 2]); HV = H * rng.choice([1, 2])
            Dk = rng.choice([1, 3, 8, 16, 33, 64, 100, 128]); Dv = rng.choice([1, 5, 16, 32, 40, 64, 100, 128])
            C = rng.choice([1, 7, 16, 32, 64]); T = rng.randint(0, 150); B = rng.choice([1, 2])
            flags = rng.random() < 0.7
            gate = rng.choice(["bounded", "softplus"]) if flags else "bounded"
            per_head = rng.random() < 0.3 if flags else False
            dtype = rng.choice(["f32", "bf16"])
            if Dk * Dv > 128 * 128 or (Dk == 1 and flags):
                continue
            case = (B, T, H, HV, Dk, Dv, C, dtype, flags, rng.choice([1.0, 0.5]), rng.randint(0, 1000), gate, per_head)
            e = R.run_case(lib, *case)
        elif kind == "step":
            H = rng.choice([1, 2]); HV = H * rng.choice([1, 2])
            Dk = rng.choice([4, 16, 64, 128]); Dv = rng.choice([4, 16, 64, 128])
            case = (rng.choice([1, 3]), H, HV, Dk, Dv, rng.choice(["f32", "bf16"]), rng.choice(["bounded", "softplus"]),
                    rng.random() < 0.3, rng.randint(0, 1000))
            e = R.run_step_case(lib, *case)
        elif kind == "compose":
            case = (rng.randint(0, 6), rng.randint(1, 3), rng.choice([1, 8, 33, 128]), rng.choice([1, 16, 40, 128]),
                    rng.random() < 0.5, rng.randint(0, 1000))
            e = R.run_compose_case(lib, *case)
        elif kind == "layer":
            case = (rng.choice([1, 2]), rng.randint(0, 140), 128 * rng.choice([1, 2]), rng.randint(1, 4),
                    rng.choice([0, 128]), rng.random() < 0.7, rng.random() < 0.5, rng.randint(0, 1000))
            e = R.run_layer_case(lib, *case)
        else:
            H = rng.choice([1, 2]); HV = H * rng.choice([1, 2])
            case = (rng.choice([1, 2]), rng.randint(1, 200), H, HV, rng.random() < 0.3, rng.choice([None, 0.05]),
                    rng.choice([0.0, -4.0, 6.0]), rng.randint(0, 1000), rng.random() < 0.3, rng.random() < 0.3)
            e = R.run_tc_case(lib, *case)
        n += 1
        worst = max(e.values()) if e else 0.0
        if worst > R.TOL:
            bad += 1
            print("MISMATCH", kind, case, e, flush=True)
    except Exception as ex:
        bad += 1
        print("ERROR", kind, ex, flush=True)
print("done", n, "cases", bad, "bad", flush=True)
