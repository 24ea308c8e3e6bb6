"""The oracle pins catch plausible mistakes in the oracle.

Each case plants one mistake in a temporary copy of the oracle's C source (a flipped tie rule, a
dropped term, a wrong index, bias, group size or rounding mode), and runs the oracle pins
(test_oracle_pins.py, and test_sharding.py for the expert-parallel shares) against that copy,
which rebuilds itself on first use. Every case must make at least one pin fail. The oracle under
test is never modified: the copies live in temporary folders.

The planted mistakes cover every step the oracle restates: routing (tie rule, renormalisation,
softmax scale), alignment (pad values, block rounding, slot order), the INT4, E2M1, MXFP4, NVFP4,
bf16 and E4M3 codecs, the SiLU and the gate/up row layout, the bf16 and FP8 intermediates, the
NVFP4 tensor scales, the combine weights, the block-FP8 scale indexing of the layer and the dense
matmul, the channelwise scales, the grouped GEMM's expert and padding rows, and the
expert-parallel range."""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

# (name, text in moe_oracle.c, replacement)
MUTATIONS = [
    ("route: ties to the higher index", "l[e] > l[best]) best = e;", "l[e] >= l[best]) best = e;"),
    ("route: weights not renormalised", "- lmax) / den);", "- lmax));"),
    ("route: softmax of twice the logits", "exp((double)l[ids[(size_t)t * k + j]] - lmax) / den",
     "exp(2.0 * ((double)l[ids[(size_t)t * k + j]] - lmax)) / den"),
    ("align: pad value -1", "for (long i = 0; i < cap; ++i) sorted_ids[i] = (int32_t)n;",
     "for (long i = 0; i < cap; ++i) sorted_ids[i] = -1;"),
    ("align: unused blocks hold expert 0", "for (long b = 0; b < nblk; ++b) expert_ids[b] = -1;",
     "for (long b = 0; b < nblk; ++b) expert_ids[b] = 0;"),
    ("align: an extra block on exact multiples", "long padded = (cnt[e] + B - 1) / B * B;",
     "long padded = (cnt[e] + B) / B * B;"),
    ("align: slots in descending order", "for (long f = 0; f < n; ++f)\n            if (ids[f] == e)",
     "for (long f = n - 1; f >= 0; --f)\n            if (ids[f] == e)"),
    ("INT4: zero point 7", "return (double)(code - 8) * bf16_value", "return (double)(code - 7) * bf16_value"),
    ("INT4: nibbles in reverse order", "int code = (int)((word >> (4 * (c % 8))) & 15u);",
     "int code = (int)((word >> (4 * (7 - c % 8))) & 15u);"),
    ("INT4: scale groups of 64", "bf16_value(s[(size_t)r * (K / 32) + c / 32]);",
     "bf16_value(s[(size_t)r * (K / 32) + c / 64]);"),
    ("E2M1: subnormal step 1", ": 0.5 * (double)m;", ": 1.0 * (double)m;"),
    ("E2M1: exponent bias 2", "ldexp(1.0 + 0.5 * (double)m, (int)e - 1)", "ldexp(1.0 + 0.5 * (double)m, (int)e - 2)"),
    ("MXFP4: scale bias 128", "c / 32] - 127);", "c / 32] - 128);"),
    ("NVFP4: scale groups of 32", "e4m3_value(s[(size_t)r * (K / 16) + c / 16]);",
     "e4m3_value(s[(size_t)r * (K / 16) + c / 32]);"),
    ("SiLU is the sigmoid", "static double silu(double g) { return g / (1.0 + exp(-g)); }",
     "static double silu(double g) { return 1.0 / (1.0 + exp(-g)); }"),
    ("gate read from the up rows", "g += xd[c] * q4_value(fmt, q13, s13, H, n, c);",
     "g += xd[c] * q4_value(fmt, q13, s13, H, I + n, c);"),
    ("4-bit intermediate not rounded to bf16", "h[n] = bf16_value(hb);", "h[n] = silu(g) * u;"),
    ("NVFP4: gate/up tensor scale on the gate only", "u *= ts13;", "u *= 1.0;"),
    ("NVFP4: down tensor scale dropped", "o[m] += wj * ts2 * y;", "o[m] += wj * y;"),
    ("4-bit combine weight dropped", "o[m] += wj * ts2 * y;", "o[m] += ts2 * y;"),
    ("E4M3: exponent bias 8", "else v = ldexp(1.0 + m / 8.0, e - 7);", "else v = ldexp(1.0 + m / 8.0, e - 8);"),
    ("E4M3: ties away from zero", "int r = (int)nearbyint(2.0 * m * 8.0);", "int r = (int)floor(2.0 * m * 8.0 + 0.5);"),
    ("E4M3: overflow to NaN", "if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);",
     "if (a >= 448.0) return (uint8_t)(sign | 0x7Fu);"),
    ("E4M3: subnormal ties away from zero", "int r = (int)nearbyint(a * 512.0);", "int r = (int)floor(a * 512.0 + 0.5);"),
    ("FP8 quantizer: scale amax / 447", "/ 448.0f;   /* IEEE f32 division */", "/ 447.0f;   /* IEEE f32 division */"),
    ("FP8 quantizer: zero-group floor 1e-6", "(amax > 1e-10f ? amax : 1e-10f)", "(amax > 1e-6f ? amax : 1e-6f)"),
    ("FP8 intermediate rounded to bf16", "a[n] = (float)(silu(g) * u);", "a[n] = (float)bf16_value(bf16_round(silu(g) * u));"),
    ("block FP8: weight scale of the first K block", "acc += (double)as[kb] * (double)bs[kb] * part;",
     "acc += (double)as[kb] * (double)bs[0] * part;"),
    ("block FP8: activation scale of the first K block", "acc += (double)as[kb] * (double)bs[kb] * part;",
     "acc += (double)as[0] * (double)bs[kb] * part;"),
    ("FP8 layer: gate/up scales of the first row block", "S13 + (size_t)(n / 128) * (H / 128), H);", "S13, H);"),
    ("FP8 layer: down scale rows of 256", "S2 + (size_t)(m / 128) * (I / 128), I);",
     "S2 + (size_t)(m / 256) * (I / 128), I);"),
    ("FP8 layer: combine weight dropped", "o[m] += wj * fp8_row_dot(hq, hs,", "o[m] += fp8_row_dot(hq, hs,"),
    ("dense block FP8: weight scale row n % 128", "Bs + (size_t)(n / 128) * KB, K);",
     "Bs + (size_t)(n % 128 / 128) * KB, K);"),
    ("channelwise: weight scale dropped", "C[(size_t)i * N + n] = (double)As[m] * (double)Bs[n] * dot;",
     "C[(size_t)i * N + n] = (double)As[m] * dot;"),
    ("channelwise: weight scale indexed by the row", "C[(size_t)i * N + n] = (double)As[m] * (double)Bs[n] * dot;",
     "C[(size_t)i * N + n] = (double)As[m] * (double)Bs[m % N] * dot;"),
    ("grouped: every row on expert 0", "const int32_t *q = wq + (size_t)e * N * (K / 8);", "const int32_t *q = wq;"),
    ("grouped: padding rows computed", "if (e >= 0 && e < G) {", "if (e < G) { if (e < 0) e = 0;"),
    ("bf16: ties away from zero", "double r = nearbyint(m * 256.0);", "double r = floor(m * 256.0 + 0.5);"),
    ("bf16: rounded twice through f32", "uint16_t sign = signbit(v) ? 0x8000u : 0u;\n    double a = fabs(v);",
     "uint16_t sign = signbit(v) ? 0x8000u : 0u;\n    double a = fabs((double)(float)v);"),
    ("expert parallel: experts below the range taken as the first held",
     "if (e < 0 || e >= ep_local) continue;\n            const int32_t *q13",
     "if (e < 0) e = 0;\n            if (e >= ep_local) continue;\n            const int32_t *q13"),
]

PINS = ["tests/test_oracle_pins.py", "tests/test_sharding.py"]


def _copy_tree(dst):
    """The files the pins need: the oracle (without its built library), the tests, the input
    generators and the pure-Python sharding module of the package."""
    ign = shutil.ignore_patterns("__pycache__", "*.so", "_build", "csrc")
    for d in ("oracle", "tests", "quantized_mixture_experts_align_b200"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(dst, d), ignore=ign)
    shutil.copy(os.path.join(ROOT, "workloads.py"), dst)


def _run(src, mutation):
    name, old, new = mutation
    tmp = tempfile.mkdtemp(prefix="oracle_mutation_")
    try:
        _copy_tree(tmp)
        with open(os.path.join(tmp, "oracle", "moe_oracle.c"), "w") as f:
            f.write(src.replace(old, new, 1))
        env = dict(os.environ, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-m", "not gpu", "-x", "-q", "-p", "no:cacheprovider"],
                           cwd=tmp, env=env, capture_output=True, text=True, timeout=900)
        failed = [ln for ln in r.stdout.splitlines() if ln.startswith("FAILED")]
        return name, r.returncode, failed
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def test_every_planted_mistake_fails_a_pin():
    with open(SRC) as f:
        src = f.read()
    missing = [name for name, old, _ in MUTATIONS if old not in src]
    assert not missing, f"mutation sites no longer in the oracle source: {missing}"
    workers = max(1, min(4, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(workers) as pool:
        results = list(pool.map(lambda m: _run(src, m), MUTATIONS))
    survivors = [name for name, rc, _ in results if rc == 0]
    broken = [(name, rc) for name, rc, failed in results if rc != 0 and not failed]
    assert not broken, f"pin runs that ended without a failing pin (collection or build error?): {broken}"
    assert not survivors, f"planted mistakes that no pin catches: {survivors}"
