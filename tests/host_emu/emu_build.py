"""Host emulation of the library's SIMT kernels -- TEST INFRASTRUCTURE.

Compiles the CUDA sources of the library's kernels -- the SIMT chunk forward
(kda_chunk_simt.cu), the backward (kda_chunk_bwd.cu), the decode step
(kda_step.cu), the segment combine (kda_compose.cu), the layer prologue and
epilogue (kda_layer.cu) and the tensor-core chunk kernel (kda_chunk_tc.cu,
against tcinc/tc_ptx.cuh, a host model of the tcgen05 / TMA / mbarrier
instructions it uses) -- as host C++ with g++ and AddressSanitizer: the
stand-in headers in fakeinc/ map the CUDA keywords and intrinsics the kernels
use onto C++, emu_rt.cpp runs every CUDA thread of a block as a std::thread
(__syncthreads and __syncwarp are std::barriers, a thread that returns drops
out of them as an exited GPU thread does), and the dynamic shared memory is an
array whose bytes past the launch's size are poisoned.  A kernel that reads or
writes outside its buffers, global or shared, stops with an AddressSanitizer
report.  Only the kernels are compiled: the source is cut before its host
launchers.  The library never uses any of this; the GPU tests are the parity
tests proper.
"""
import os
import re
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
CSRC = os.path.join(ROOT, "gated_delta_rule_157_b200", "csrc")
OUT = os.path.join(HERE, "_build")
LIB = os.path.join(OUT, "libkda_host_emu.so")
SMEM_FLOATS = 65536

# extern "C" runners appended to each unit: the grid and block of the
# library's launchers, with the shared-memory bytes poisoned past the size the
# kernel asks for.
_POISON = r'''
#include <sanitizer/asan_interface.h>
namespace kda { namespace {
void emu_poison(size_t used) {
    ASAN_UNPOISON_MEMORY_REGION(smem, sizeof(smem));
    ASAN_POISON_MEMORY_REGION(reinterpret_cast<char *>(smem) + used, sizeof(smem) - used);
}
} }
'''
_RUN_FWD = _POISON + r'''
extern "C" int emu_sizeof_chunk_params(void) { return (int)sizeof(kda::ChunkParams); }
extern "C" int emu_offsetof_withhold_ready(void) { return (int)offsetof(kda::ChunkParams, withhold_ready); }
extern "C" int emu_chunk_fwd(kda::ChunkParams *pp, int bf16) {
    using namespace kda;
    const ChunkParams p = *pp;
    const int ncol = p.Dv + (p.M_T ? p.Dk : 0);
    const size_t bytes = simt_smem_bytes(p.C, p.Dk);
    if (bytes > sizeof(smem)) return 1;
    emu_poison(bytes);
    const dim3 grid(p.B * p.HV, (ncol + kVT - 1) / kVT);
    if (bf16) emu_launch(grid, dim3(kThreads), [&] { chunk_simt_kernel<__nv_bfloat16>(p); });
    else emu_launch(grid, dim3(kThreads), [&] { chunk_simt_kernel<float>(p); });
    return 0;
}
'''
_RUN_BWD = _POISON + r'''
extern "C" int emu_sizeof_bwd_params(void) { return (int)sizeof(kda::BwdParams); }
extern "C" int emu_offsetof_ddt_bias(void) { return (int)offsetof(kda::BwdParams, ddt_bias); }
template <typename Tin>
static void run_bwd(const kda::BwdParams &p) {
    using namespace kda;
    if (bwd_anchored(p))
        emu_launch(dim3(p.B * p.HV, (p.Dv + kVT - 1) / kVT), dim3(kThreads), [&] { chunk_bwd_kernel<Tin, true>(p); });
    else
        emu_launch(dim3(p.B * p.HV, (p.Dv + kVT - 1) / kVT), dim3(kThreads), [&] { chunk_bwd_kernel<Tin, false>(p); });
    emu_poison(0);
    if (p.l2norm) {
        const long long rows = (long long)p.B * p.T * p.H;
        emu_launch(dim3((unsigned)((rows + kRowThreads / 32 - 1) / (kRowThreads / 32))), dim3(kRowThreads),
                   [&] { bwd_l2norm_kernel<Tin>(p); });
    }
    if (p.beta_sigmoid || p.gate_in) {
        const long long ntok = (long long)p.B * p.T;
        emu_launch(dim3(p.HV, (unsigned)((ntok + kGateTokens - 1) / kGateTokens)), dim3(128),
                   [&] { bwd_gate_kernel<Tin>(p); });
    }
}
// The outputs the library zeroes before these kernels must arrive zeroed.
extern "C" int emu_chunk_bwd(kda::BwdParams *pp, int bf16) {
    using namespace kda;
    const BwdParams p = *pp;
    const size_t bytes = bwd_smem_bytes(p.C, p.Dk, bwd_anchored(p));
    if (bytes > sizeof(smem)) return 1;
    emu_poison(bytes);
    if (p.T == 0) {
        emu_poison(0);
        emu_launch(dim3(2), dim3(64), [&] { bwd_empty_kernel(p); });
        return 0;
    }
    if (bf16) run_bwd<__nv_bfloat16>(p);
    else run_bwd<float>(p);
    return 0;
}
'''


_RUN_TC = r'''
#include <sanitizer/asan_interface.h>
namespace kda { namespace tc { EmuCta *g_cta = nullptr; EmuTf32Slots g_tf32[32]; } }

// The tensor maps the library's launcher builds (tokens x heads x 128 channels,
// [64][1][128] boxes; v in two [64][1][64] boxes with the 128-byte swizzle).
static kda::tc::EmuTensorMap emu_row_map(const void *base, int heads, long long rows, bool sw128) {
    kda::tc::EmuTensorMap m{};
    m.base = static_cast<const uint8_t *>(base);
    m.dims[0] = 128; m.dims[1] = (uint64_t)heads; m.dims[2] = (uint64_t)rows;
    m.strides[0] = 128 * 2; m.strides[1] = (uint64_t)heads * 128 * 2;
    m.box[0] = sw128 ? 64 : 128; m.box[1] = 1; m.box[2] = 64;
    m.swizzle128 = sw128 ? 1 : 0;
    return m;
}

extern "C" int emu_chunk_tc(kda::ChunkParams *pp) {
    using namespace kda;
    TcParams tp;
    tp.p = *pp;
    const long long rows = (long long)tp.p.B * tp.p.T;
    const tc::EmuTensorMap maps[4] = {emu_row_map(tp.p.q, tp.p.H, rows, false), emu_row_map(tp.p.k, tp.p.H, rows, false),
                                      emu_row_map(tp.p.g, tp.p.HV, rows, false),
                                      emu_row_map(tp.p.v, tp.p.HV, rows, true)};
    for (int i = 0; i < 4; ++i) std::memcpy(&tp.tm[i], &maps[i], sizeof maps[i]);
    const tc::EmuTensorMap omap = emu_row_map(tp.p.o, tp.p.HV, rows, false);
    std::memcpy(&tp.tm[4], &omap, sizeof omap);
    tp.o_tma = tp.p.o ? 1 : 0;
    static tc::EmuCta cta;
    static tc::EmuMBar bars[sizeof smem_raw / 8];
    cta.smem = smem_raw;
    cta.smem_bytes = SMEM_BYTES;
    cta.bars = bars;
    g_device_error = 0;
    emu_launch_cb(dim3(tp.p.B * tp.p.HV, tp.p.M_T ? 2 : 1), dim3(kThreads),
                  [&](unsigned, unsigned) {
                      ASAN_UNPOISON_MEMORY_REGION(smem_raw, sizeof smem_raw);
                      std::memset(cta.tmem, 0, sizeof cta.tmem);
                      std::memset(smem_raw, 0, sizeof smem_raw);
                      ASAN_POISON_MEMORY_REGION(smem_raw + SMEM_BYTES, sizeof smem_raw - SMEM_BYTES);
                      tc::g_cta = &cta;
                  },
                  [&] { chunk_tc_kernel(tp); });
    return g_device_error ? 2 : 0;
}
'''


def _tc_unit(runner=_RUN_TC):
    """The tensor-core chunk kernel against the host model of its PTX wrappers
    (tcinc/tc_ptx.cuh, found before the library's own): the source up to its
    host functions, the 240 KB shared array, and the runner above."""
    s = open(os.path.join(CSRC, "kda_chunk_tc.cu")).read()
    s = s[: s.index("bool chunk_tc_supported")] + "}  // namespace kda\n"
    s = s.replace("extern __shared__", "extern").replace("__shared__", "static")
    head = ('#include <functional>\n#include "cuda_runtime.h"\n'
            "void emu_launch_cb(dim3 grid, dim3 block, const std::function<void(unsigned, unsigned)> &on_block,\n"
            "                   const std::function<void()> &fn);\n"
            "namespace kda { namespace { alignas(1024) uint8_t smem_raw[240 * 1024]; } }\n")
    return head + '#line 1 "kda_chunk_tc.cu"\n' + s + runner


def unit_from_text(text, runner, poison=True):
    """A unit for kernel source text given directly (namespace kda, unnamed
    namespace, no host launchers): the checks of the harness itself."""
    head = ('#include <functional>\n#include "cuda_runtime.h"\n'
            "void emu_launch(dim3 grid, dim3 block, const std::function<void()> &fn);\n"
            "namespace kda { namespace { alignas(16) float smem[%d]; } }\n" % SMEM_FLOATS)
    body = text.replace("extern __shared__", "extern").replace("__shared__", "static")
    return head + body + (_POISON if poison else "") + runner


def _unit(src_name, runner, src_dir=CSRC):
    s = open(os.path.join(src_dir, src_name)).read()
    m = re.search(r"^(template <[^>]*>\n(static )?)?cudaError_t launch_", s, re.M)
    if not m:
        raise RuntimeError("no host launcher found in " + src_name)
    s = s[: m.start()]
    if "\n}  // namespace\n" not in s:      # the first launcher sits inside the unnamed namespace
        s += "\n}  // namespace\n"
    s += "}  // namespace kda\n"
    # static __shared__ arrays are block-wide: function statics (the blocks of
    # a grid run one after another); the dynamic one is the array declared below
    s = s.replace("extern __shared__", "extern").replace("__shared__", "static")
    head = ('#include <functional>\n#include "cuda_runtime.h"\n'
            "void emu_launch(dim3 grid, dim3 block, const std::function<void()> &fn);\n"
            "namespace kda { namespace { alignas(16) float smem[%d]; } }\n" % SMEM_FLOATS)
    return head + "#line 1 \"%s\"\n" % src_name + s + runner


_RUN_STEP = _POISON + r'''
void emu_launch_cb(dim3 grid, dim3 block, const std::function<void(unsigned, unsigned)> &on_block,
                   const std::function<void()> &fn);
extern "C" int emu_sizeof_step_params(void) { return (int)sizeof(kda::StepParams); }
template <int RPT>
static void run_step(const kda::StepParams &p, int bf16) {
    using namespace kda;
    if (bf16) emu_launch(dim3(p.B * p.HV), dim3(kThreads), [&] { step_kernel<RPT, __nv_bfloat16>(p); });
    else emu_launch(dim3(p.B * p.HV), dim3(kThreads), [&] { step_kernel<RPT, float>(p); });
}
namespace kda { namespace tc { extern EmuCta *g_cta; } }
// Dk = Dv = 128: the persistent bulk-copy kernel, on a grid of at most two
// CTAs so that every CTA walks several chains through its stage ring.
static void run_step_bulk(const kda::StepParams &p, int bf16) {
    using namespace kda;
    static tc::EmuCta cta;
    static tc::EmuMBar bars[sizeof(smem) / 8];
    cta.smem = reinterpret_cast<uint8_t *>(smem);
    cta.smem_bytes = BULK_SMEM;
    cta.bars = bars;
    const int nchains = p.B * p.HV;
    const unsigned grid = nchains < 2 ? (unsigned)nchains : 2u;
    emu_launch_cb(dim3(grid), dim3(kThreads), [&](unsigned, unsigned) {
        emu_poison(BULK_SMEM);
        std::memset(smem, 0, BULK_SMEM);
        tc::g_cta = &cta;
    }, [&] {
        if (bf16) step_bulk_kernel<__nv_bfloat16>(p);
        else step_bulk_kernel<float>(p);
    });
}
extern "C" int emu_step(kda::StepParams *pp, int bf16) {
    const kda::StepParams p = *pp;
    if (p.Dk == 128 && p.Dv == 128) {
        run_step_bulk(p, bf16);
        return 0;
    }
    const int rpt = (p.Dk + kda::kWarps - 1) / kda::kWarps;
    if (rpt <= 1) run_step<1>(p, bf16);
    else if (rpt <= 2) run_step<2>(p, bf16);
    else if (rpt <= 4) run_step<4>(p, bf16);
    else if (rpt <= 8) run_step<8>(p, bf16);
    else run_step<16>(p, bf16);
    return 0;
}
'''


_RUN_COMPOSE = _POISON + r'''
extern "C" int emu_compose(int n_seg, int BH, int Dk, int Dv, const float *M, const float *S_seg,
                           const float *S_init, float *S_in) {
    using namespace kda;
    emu_poison(0);     // the kernel's shared memory is static
    const bool vec = Dk % 4 == 0 && Dv % 4 == 0 && ((uintptr_t)M | (uintptr_t)S_seg | (uintptr_t)S_init |
                                                    (uintptr_t)S_in) % 16 == 0;
    emu_launch(dim3(BH, (Dv + kVT - 1) / kVT), dim3(kThreads), [&] {
        if (vec) compose_kernel<true>(n_seg, BH, Dk, Dv, M, S_seg, S_init, S_in);
        else compose_kernel<false>(n_seg, BH, Dk, Dv, M, S_seg, S_init, S_in);
    });
    return 0;
}
'''
_RUN_LAYER = _POISON + r'''
void emu_launch_cb(dim3 grid, dim3 block, const std::function<void(unsigned, unsigned)> &on_block,
                   const std::function<void()> &fn);
extern "C" int emu_sizeof_conv_params(void) { return (int)sizeof(kda::ConvParams); }
extern "C" int emu_sizeof_gate_params(void) { return (int)sizeof(kda::GateParams); }
namespace kda { namespace tc { extern EmuCta *g_cta; } }
// The tiled kernel's tensor maps ([B][T][C], boxes of [1][rows][256]), run on
// a grid of at most three CTAs so that every CTA walks several tiles through
// its stage ring (and, with two or more channel groups, changes groups).
static kda::tc::EmuTensorMap emu_conv_map(const void *base, const kda::ConvParams &p, int rows) {
    kda::tc::EmuTensorMap m{};
    m.base = static_cast<const uint8_t *>(base);
    m.dims[0] = (uint64_t)p.C; m.dims[1] = (uint64_t)p.T; m.dims[2] = (uint64_t)p.B;
    m.strides[0] = (uint64_t)p.C * 2; m.strides[1] = (uint64_t)p.T * p.C * 2;
    m.box[0] = 256; m.box[1] = (uint32_t)rows; m.box[2] = 1;
    return m;
}
template <int K>
static void run_conv_tma(const kda::ConvParams &p) {
    using namespace kda;
    ConvTmaParams tp;
    tp.p = p;
    const tc::EmuTensorMap mx = emu_conv_map(p.x, p, kTT + kHalo);
    std::memcpy(&tp.tx, &mx, sizeof mx);
    static tc::EmuCta cta;
    static tc::EmuMBar bars[sizeof(smem) / 8];
    cta.smem = reinterpret_cast<uint8_t *>(smem);
    cta.smem_bytes = TS_SMEM;
    cta.bars = bars;
    const long long ntiles = (long long)p.B * (p.C / kTC) * ((p.T + kTT - 1) / kTT);
    const unsigned grid = ntiles < 3 ? (unsigned)ntiles : 3u;
    emu_launch_cb(dim3(grid), dim3(kConvThreads), [&](unsigned, unsigned) {
        emu_poison(TS_SMEM);
        std::memset(smem, 0, TS_SMEM);
        tc::g_cta = &cta;
    }, [&] { short_conv_tma_kernel<K>(tp); });
}
extern "C" int emu_short_conv(kda::ConvParams *pp) {
    using namespace kda;
    const ConvParams p = *pp;
    if (p.C % kTC == 0 && p.T > 0 && p.K >= 1 && p.K <= 4 && (p.head_dim == 0 || p.head_dim == 128) &&
        (uintptr_t)p.state_in % 16 == 0 && (uintptr_t)p.state_out % 16 == 0 && (uintptr_t)p.y % 16 == 0) {
        switch (p.K) {
            case 1: run_conv_tma<1>(p); break;
            case 2: run_conv_tma<2>(p); break;
            case 3: run_conv_tma<3>(p); break;
            default: run_conv_tma<4>(p); break;
        }
        return 0;
    }
    const long long warps = conv_grid_warps(p);
    if (warps == 0) return 0;
    const dim3 grid((unsigned)((warps + kLayerThreads / 32 - 1) / (kLayerThreads / 32)));
    switch (p.K) {
        case 1: emu_launch(grid, dim3(kLayerThreads), [&] { short_conv_kernel<1>(p); }); break;
        case 2: emu_launch(grid, dim3(kLayerThreads), [&] { short_conv_kernel<2>(p); }); break;
        case 3: emu_launch(grid, dim3(kLayerThreads), [&] { short_conv_kernel<3>(p); }); break;
        default: emu_launch(grid, dim3(kLayerThreads), [&] { short_conv_kernel<4>(p); }); break;
    }
    return 0;
}
extern "C" int emu_output_gate(kda::GateParams *pp) {
    using namespace kda;
    const GateParams p = *pp;
    const long long warps = ((long long)p.N * p.HV + kGateRows - 1) / kGateRows;
    if (warps == 0) return 0;
    emu_launch(dim3((unsigned)((warps + kLayerThreads / 32 - 1) / (kLayerThreads / 32))), dim3(kLayerThreads),
               [&] { output_gate_kernel(p); });
    return 0;
}
'''


def _deps():
    return [os.path.join(CSRC, f) for f in ("kda_chunk_simt.cu", "kda_chunk_bwd.cu", "kda_step.cu",
                                            "kda_compose.cu", "kda_layer.cu", "kda_chunk_tc.cu",
                                            "kda_internal.cuh")] + \
        [os.path.join(HERE, f) for f in ("emu_build.py", "emu_rt.cpp", "fakeinc/cuda_runtime.h", "fakeinc/cuda_bf16.h",
                                         "fakeinc/cuda.h", "tcinc/tc_ptx.cuh")] + \
        [os.path.join(ROOT, "include", "kda.h")]


def sanitizer_runtime(sanitizer="address"):
    """Path of the g++ sanitizer runtime to preload (libasan / libtsan)."""
    name = {"address": "libasan.so", "thread": "libtsan.so"}[sanitizer]
    return subprocess.run(["g++", "-print-file-name=" + name], check=True, capture_output=True,
                          text=True).stdout.strip()


def asan_runtime():
    return sanitizer_runtime("address")


def compile_units(units, lib_path, sanitizer="address", src_dir=CSRC):
    """Compile {file name: C++ text} plus the thread runtime into lib_path."""
    out = os.path.dirname(lib_path)
    os.makedirs(out, exist_ok=True)
    tag = "" if sanitizer == "address" else "." + sanitizer
    flags = ["g++", "-std=c++20", "-O1", "-g", "-fsanitize=" + sanitizer, "-fno-omit-frame-pointer", "-fPIC",
             "-I", os.path.join(HERE, "fakeinc"), "-I", os.path.join(HERE, "tcinc"), "-I", src_dir, "-I", CSRC,
             "-Wno-unknown-pragmas", "-c"]
    objs = []
    for name, text in units.items():
        path = os.path.join(out, name)
        with open(path, "w") as f:
            f.write(text)
        objs.append(path[:-4] + tag + ".o")
        subprocess.run(flags + [path, "-o", objs[-1]], check=True)
    objs.append(os.path.join(out, "emu_rt%s.o" % tag))
    subprocess.run(flags + [os.path.join(HERE, "emu_rt.cpp"), "-o", objs[-1]], check=True)
    tmp = lib_path + ".tmp.%d" % os.getpid()
    subprocess.run(["g++", "-shared", "-fsanitize=" + sanitizer, "-o", tmp, *objs, "-pthread"], check=True)
    os.replace(tmp, lib_path)
    return lib_path


def build(force=False, sanitizer="address"):
    """Compile libkda_host_emu.so (AddressSanitizer) or libkda_host_emu_tsan.so
    (ThreadSanitizer); skipped when newer than its sources."""
    lib = LIB if sanitizer == "address" else LIB[:-3] + "_tsan.so"
    if not force and os.path.exists(lib) and all(os.path.getmtime(d) <= os.path.getmtime(lib) for d in _deps()):
        return lib
    units = {"emu_fwd.cpp": _unit("kda_chunk_simt.cu", _RUN_FWD),
             "emu_bwd.cpp": _unit("kda_chunk_bwd.cu", _RUN_BWD),
             "emu_step.cpp": _unit("kda_step.cu", _RUN_STEP),
             "emu_compose.cpp": _unit("kda_compose.cu", _RUN_COMPOSE),
             "emu_layer.cpp": _unit("kda_layer.cu", _RUN_LAYER),
             "emu_tc.cpp": _tc_unit()}
    if sanitizer != "address":      # the shared-memory poisoning is AddressSanitizer's
        units = {n: t.replace("#include <sanitizer/asan_interface.h>", "#define ASAN_POISON_MEMORY_REGION(a, b)\n"
                              "#define ASAN_UNPOISON_MEMORY_REGION(a, b)") for n, t in units.items()}
    return compile_units(units, lib, sanitizer)


if __name__ == "__main__":
    print(build(force=True))
