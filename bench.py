"""Benchmark of the fine-grained online FP8 hot path on B200.

One step = one pass of the hot path over one batch of synthetic input.
Workloads (``--workload``):
  ffn    (default) dense FFN up-projection forward: X bf16 [4096x7168] and
         W bf16 [7168x18432] quantized online (1x128 / 128x128, scales
         computed on every step), block-scaled FP8 GEMM -> bf16 [4096x18432].
         3 launches per step.  value = 2MNK / step time (TFLOP/s).
  quant  quantize-only bandwidth: act [8192x7168] and weight [7168x18432]
         bf16.  value = bytes moved / step time (GB/s).
  moe    MoE expert GEMMs, 8192 tokens x top-8 of 256 experts: act quant of
         the routed tokens, grouped gate+up GEMM (N=4096, K=7168), act quant
         of the down input, grouped down GEMM (N=7168, K=2048).  Expert
         weights are quantized once before timing.  value in TFLOP/s.
  dgrad  backward dgrad: dY bf16 [16384x18432] quantized 1x128 along N, W
         [7168x18432] quantized (untransposed), dX = dY W^T -> bf16.
  wgrad  backward wgrad: X bf16 [16384x7168] and dY bf16 [16384x18432]
         quantized in 1x128 tiles along the 16384 tokens (written transposed),
         dW = X^T dY -> fp32 [7168x18432] by the GEMM with per-column B scales.
  ffn_q  ffn with the GEMM's output quantized 1x128 in its epilogue.
  dequant  the FFN weight's codes back to bf16.

Contract: ``python bench.py --gpus N --steps K --warmup W`` (N > 1 under
torchrun, one rank per GPU) prints one JSON line on rank 0.  Each rank runs
its own replica of the workload (data parallel over tokens: no collective on
the data path); the time is the max over ranks of the CUDA-event time of K
steps, taken between barriers and device synchronizations.
``--impl reference`` times the plain CPU oracle instead, on a bounded
sample of the same workload (rank 0 only).
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "FP8 block-scaled GEMM TFLOP/s & quantize GB/s, % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0     # nominal dense ratio, 4.5 / 2.25 PFLOP/s
CSRC = os.path.join(ROOT, "fp8_fine_grained_online_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")
QUEUE_FILL_CYCLES = 400_000   # ~0.2 ms of device spin ahead of a timed region


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    """The measured HBM copy and bf16 GEMM peaks when MEASURED_PEAKS.json is
    present and holds them as numbers, else the fallback figures."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            with open(path) as f:
                d = json.load(f)
            if all(isinstance(d.get(k), (int, float)) and d[k] > 0
                   for k in ("hbm_gbs", "bf16_tflops")):
                out = dict(FALLBACK_PEAKS)
                out.update({k: float(v) for k, v in d.items()
                            if k in FALLBACK_PEAKS and isinstance(v, (int, float)) and v > 0})
                return out, "measured"
        except (OSError, ValueError, AttributeError):
            pass
    return dict(FALLBACK_PEAKS), "fallback"


def _strip_comments(src):
    """C/C++ source without its comments and trailing blanks (string
    literals holding comment markers do not occur in the kernel sources)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_source_hash():
    """Hash of the kernel sources' code (comments and blank lines ignored),
    the key under which profiles/dram_traffic.txt records its counters."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            h.update(name.encode() + _strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    cur = kernel_source_hash()
    with open(TRAFFIC_FILE) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#"):
                k, w, b, src_hash = parts[:4]
                if k == kernel and w == workload and src_hash == cur:
                    return float(b)
    return None


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region.

    NVML (read-only queries) from a background thread every ~2 ms, so that
    even a timed region of a few milliseconds gets several samples; the GPU
    is found by its PCI address (robust to CUDA_VISIBLE_DEVICES).  Falls back
    to `nvidia-smi -lms 100` when NVML is not importable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_S = 0.002

    def __init__(self, device_index):
        import threading
        self.proc = None
        self.thread = None
        self.samples = []
        self.reasons = set()
        try:
            import pynvml
            pynvml.nvmlInit()
            prop = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (prop.pci_domain_id, prop.pci_bus_id, prop.pci_device_id)
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.reason_bits = {
                "hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            self.stop_flag = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(device_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def _poll(self):
        n = self.nvml
        while not self.stop_flag.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM))
                bits = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                for name, bit in self.reason_bits.items():
                    if bits & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.INTERVAL_S)

    def begin(self):
        """Start of the timed region: drop samples taken before it."""
        self.samples = []
        self.reasons = set()

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": float(self.max_mhz),
                    "reasons": sorted(self.reasons), "samples": len(self.samples),
                    "source": "nvml, every %.0f ms" % (self.INTERVAL_S * 1e3)}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, every 100 ms"}


# ----------------------------------------------------------------------------- workloads

class Workload:
    name = ""
    unit = "TFLOP/s"
    dominant = ""

    def launches_per_step(self):
        return len(self.kernels)

    def work_per_step(self):
        """Units of `value` per step (FLOP or bytes)."""
        raise NotImplementedError

    def e2e_join(self, stream):
        """Make `stream` wait for every e2e step submitted (a no-op when the
        steps run on `stream` itself)."""

    def e2e_teardown(self):
        """Drop the pinned host copies made by e2e_setup."""
        for k in list(vars(self)):
            v = getattr(self, k)
            if isinstance(v, torch.Tensor) and not v.is_cuda and k.startswith("h"):
                delattr(self, k)


def error_vs_exact(c, exact, sample):
    """Quantization error of the FP8 path against the unquantized product,
    both fp64 tensors of the same sampled entries: max|C - E| / max|E| and
    the relative Frobenius error ||C - E|| / ||E||."""
    d = c - exact
    return {"max_rel": float(d.abs().max() / exact.abs().max()),
            "fro_rel": float(torch.linalg.norm(d) / torch.linalg.norm(exact)),
            "entries": int(exact.numel()), "sample": sample}


def sample_index(n, count, device):
    """`count` indices spread evenly over range(n) (all of them if n <= count)."""
    count = min(n, count)
    return (torch.arange(count, device=device, dtype=torch.int64) * n) // count


def quant_error_tiny(fp8, device):
    """The tiny end-to-end config in full: A fp32 [128x256], B fp32 [256x256]
    quantized (1x128 / 128x128), block-scaled GEMM -> fp32, against the fp64
    product of the unquantized A and B."""
    a, b = synth.tiny_inputs(device)
    qa, sa = fp8.fp8_quantize_act_1x128(a)
    qb, sb = fp8.fp8_quantize_weight_128x128(b, transpose_out=True)
    c = fp8.fp8_blockscaled_gemm(qa, sa, qb, sb, out_dtype=torch.float32)
    exact = a.double() @ b.double()
    return error_vs_exact(c.double(), exact, "all 128 x 256 entries")


class FFN(Workload):
    """Online-quantized dense FFN up-projection forward."""
    name = synth.FFN.name
    unit = "TFLOP/s"
    dominant = "blockscaled_gemm"

    def __init__(self, fp8, device, M=4096, K=7168, N=18432):
        self.fp8, self.M, self.K, self.N = fp8, M, K, N
        self.kernels = ["quant_act_1x128", "quant_weight_128x128", "blockscaled_gemm"]
        if device is None:
            return
        self.x, self.w = synth.ffn_inputs(device, M, K, N)
        self.qx = torch.empty((M, K), dtype=torch.uint8, device=device)
        self.sx = torch.empty((M, K // 128), dtype=torch.float32, device=device)
        self.qw = torch.empty((N, K), dtype=torch.uint8, device=device)
        self.sw = torch.empty((K // 128, N // 128), dtype=torch.float32, device=device)
        self.c = torch.empty((M, N), dtype=torch.bfloat16, device=device)

    def config(self):
        return {"workload": self.name, "M": self.M, "N": self.N, "K": self.K,
                "x": "bf16 [%dx%d] N(0,1) 0.1%% outliers x100" % (self.M, self.K),
                "w": "bf16 [%dx%d] N(0,0.02)" % (self.K, self.N), "out": "bf16",
                "l2": "inputs larger than L2 (X+W bf16 = %.0f MB > 126 MB)" %
                      ((self.M * self.K + self.K * self.N) * 2 / 1e6)}

    def flops(self):
        return 2.0 * self.M * self.N * self.K

    def work_per_step(self):
        return self.flops()

    def algorithmic(self):
        """Per launch: (kind, amount) -- bytes for HBM-bound kernels, FLOPs for the GEMM."""
        M, N, K = self.M, self.N, self.K
        return {
            "quant_act_1x128": ("bytes", M * K * 2 + M * K + M * (K // 128) * 4),
            "quant_weight_128x128": ("bytes", K * N * 2 + K * N + (K // 128) * (N // 128) * 4),
            "blockscaled_gemm": ("flops", 2.0 * M * N * K),
        }

    def step(self, marks):
        f = self.fp8
        marks(0)
        f.fp8_quantize_act_1x128(self.x, q=self.qx, sa=self.sx)
        marks(1)
        f.fp8_quantize_weight_128x128(self.w, transpose_out=True, q=self.qw, sb=self.sw)
        marks(2)
        f.fp8_blockscaled_gemm(self.qx, self.sx, self.qw, self.sw, c=self.c)
        marks(3)

    def quant_error(self, rows=256, blocks=16):
        """Last step's bf16 C on a spread sample of rows x 128-column blocks
        against the fp64 product of the unquantized bf16 X and W."""
        dev = self.c.device
        r = sample_index(self.M, rows, dev)
        nb = sample_index(self.N // 128, blocks, dev)
        cols = (nb[:, None] * 128 + torch.arange(128, device=dev)).reshape(-1)
        exact = self.x[r].double() @ self.w[:, cols].double()
        return error_vs_exact(self.c[r][:, cols].double(), exact,
                              "%d rows x %d 128-column blocks, spread evenly" % (len(r), len(nb)))

    # end to end through the public API with pinned host buffers
    def e2e_setup(self):
        self.hx = self.x.cpu().pin_memory()
        self.hw = self.w.cpu().pin_memory()
        self.hc = torch.empty((self.M, self.N), dtype=torch.bfloat16, pin_memory=True)
        self.pipe = self.fp8.LinearForwardPipeline(self.M, self.K, self.N)
        return self.hx.numel() * 2 + self.hw.numel() * 2, self.hc.numel() * 2

    def e2e_step(self):
        # pipelined across steps: step i's result travels back while step
        # i+1's inputs travel in (separate copy streams, both link directions)
        self.pipe.submit(self.hx, self.hw, self.hc)

    def e2e_join(self, stream):
        if getattr(self, "pipe", None) is not None:   # subclasses run their steps on `stream`
            self.pipe.join(stream)

    def e2e_teardown(self):
        if getattr(self, "pipe", None) is not None:
            self.pipe.close()
            self.pipe = None
        Workload.e2e_teardown(self)

    def oracle_sample(self, orc, rows, nbs):
        """Oracle on a sample of the step: quantize `rows` rows of X and the
        `nbs` 128-column blocks of W, GEMM those rows x columns.  Returns the
        FLOPs of the sampled GEMM (the unit the step is counted in)."""
        xs = synth.ffn_inputs("cpu", M=self.M, K=self.K, N=self.N) if not hasattr(self, "_cpu") \
            else self._cpu
        self._cpu = xs
        x, w = xs
        xa = x[:rows].contiguous().view(torch.int16).numpy().view(np.uint16)
        qa, sa = orc.quantize_act_1x128(xa)
        flops = 0.0
        for nb in range(nbs):
            blk = w[:, nb * 128:(nb + 1) * 128].contiguous().view(torch.int16).numpy().view(np.uint16)
            qb, sb = orc.quantize_weight_128x128(blk, transpose_out=True)
            orc.gemm_ref(qa, sa, qb, sb)
            flops += 2.0 * rows * 128 * self.K
        return flops


class FFNQuantOut(FFN):
    """The FFN forward with its output quantized in the GEMM epilogue for the
    next layer (E4M3 codes + 1x128 scales instead of a bf16 C)."""
    name = "ffn_up_fwd_4096x18432x7168_fp8_out"
    dominant = "blockscaled_gemm_quant"

    def __init__(self, fp8, device, M=4096, K=7168, N=18432):
        super().__init__(fp8, device, M, K, N)
        self.kernels = ["quant_act_1x128", "quant_weight_128x128", "blockscaled_gemm_quant"]
        if device is None:
            return
        del self.c
        self.qc = torch.empty((M, N), dtype=torch.uint8, device=device)
        self.sc = torch.empty((M, N // 128), dtype=torch.float32, device=device)

    def config(self):
        d = super().config()
        d["workload"] = self.name
        d["out"] = "E4M3 [%dx%d] + fp32 1x128 scales (quantized in the GEMM epilogue)" % (self.M, self.N)
        return d

    quant_error = None     # no bf16 C is kept (the ffn workload reports it)

    def algorithmic(self):
        d = super().algorithmic()
        d["blockscaled_gemm_quant"] = d.pop("blockscaled_gemm")
        return d

    def step(self, marks):
        f = self.fp8
        marks(0)
        f.fp8_quantize_act_1x128(self.x, q=self.qx, sa=self.sx)
        marks(1)
        f.fp8_quantize_weight_128x128(self.w, transpose_out=True, q=self.qw, sb=self.sw)
        marks(2)
        f.fp8_blockscaled_gemm_quant(self.qx, self.sx, self.qw, self.sw, qc=self.qc, sc=self.sc)
        marks(3)

    def e2e_setup(self):
        self.hx = self.x.cpu().pin_memory()
        self.hw = self.w.cpu().pin_memory()
        self.hqc = torch.empty((self.M, self.N), dtype=torch.uint8, pin_memory=True)
        self.hsc = torch.empty((self.M, self.N // 128), dtype=torch.float32, pin_memory=True)
        return self.hx.numel() * 2 + self.hw.numel() * 2, self.hqc.numel() + self.hsc.numel() * 4

    def e2e_step(self):
        f = self.fp8
        x = self.hx.to("cuda", non_blocking=True)
        w = self.hw.to("cuda", non_blocking=True)
        qx, sx = f.fp8_quantize_act_1x128(x)
        qw, sw = f.fp8_quantize_weight_128x128(w, transpose_out=True)
        qc, sc = f.fp8_blockscaled_gemm_quant(qx, sx, qw, sw)
        self.hqc.copy_(qc, non_blocking=True)
        self.hsc.copy_(sc, non_blocking=True)

    def oracle_sample(self, orc, rows, nbs):
        """As FFN's, plus the 1x128 quantization of each sampled bf16 output block."""
        xs = synth.ffn_inputs("cpu", M=self.M, K=self.K, N=self.N) if not hasattr(self, "_cpu") \
            else self._cpu
        self._cpu = xs
        x, w = xs
        xa = x[:rows].contiguous().view(torch.int16).numpy().view(np.uint16)
        qa, sa = orc.quantize_act_1x128(xa)
        flops = 0.0
        for nb in range(nbs):
            blk = w[:, nb * 128:(nb + 1) * 128].contiguous().view(torch.int16).numpy().view(np.uint16)
            qb, sb = orc.quantize_weight_128x128(blk, transpose_out=True)
            c_ref, _ = orc.gemm_ref(qa, sa, qb, sb, want_t=False)
            orc.quantize_act_1x128(orc.f32_to_bf16_bits(c_ref.astype(np.float32)))
            flops += 2.0 * rows * 128 * self.K
        return flops


class Quant(Workload):
    name = synth.QUANT.name
    unit = "GB/s"
    dominant = "quant_weight_128x128"

    def __init__(self, fp8, device, M=8192, K=7168, N=18432):
        self.fp8, self.M, self.K, self.N = fp8, M, K, N
        self.kernels = ["quant_act_1x128", "quant_weight_128x128"]
        if device is None:
            return
        self.x, self.w = synth.quant_inputs(device)
        self.qx = torch.empty((M, K), dtype=torch.uint8, device=device)
        self.sx = torch.empty((M, K // 128), dtype=torch.float32, device=device)
        self.qw = torch.empty((N, K), dtype=torch.uint8, device=device)
        self.sw = torch.empty((K // 128, N // 128), dtype=torch.float32, device=device)

    def config(self):
        return {"workload": self.name, "act": "bf16 [%dx%d]" % (self.M, self.K),
                "weight": "bf16 [%dx%d] -> E4M3 [N,K]" % (self.K, self.N),
                "dist": "N(0,0.02), 0.1% outliers x100",
                "l2": "weight input 264 MB > L2; the weight pass evicts the act input"}

    def algorithmic(self):
        M, N, K = self.M, self.N, self.K
        return {
            "quant_act_1x128": ("bytes", M * K * 2 + M * K + M * (K // 128) * 4),
            "quant_weight_128x128": ("bytes", K * N * 2 + K * N + (K // 128) * (N // 128) * 4),
        }

    def work_per_step(self):
        return sum(v for _, v in self.algorithmic().values())

    def step(self, marks):
        f = self.fp8
        marks(0)
        f.fp8_quantize_act_1x128(self.x, q=self.qx, sa=self.sx)
        marks(1)
        f.fp8_quantize_weight_128x128(self.w, transpose_out=True, q=self.qw, sb=self.sw)
        marks(2)

    def e2e_setup(self):
        self.hx = self.x.cpu().pin_memory()
        self.hw = self.w.cpu().pin_memory()
        self.hqx = torch.empty_like(self.qx, device="cpu").pin_memory()
        self.hqw = torch.empty_like(self.qw, device="cpu").pin_memory()
        self.hsx = torch.empty_like(self.sx, device="cpu").pin_memory()
        self.hsw = torch.empty_like(self.sw, device="cpu").pin_memory()
        return ((self.hx.numel() + self.hw.numel()) * 2,
                self.hqx.numel() + self.hqw.numel() + (self.hsx.numel() + self.hsw.numel()) * 4)

    def e2e_step(self):
        f = self.fp8
        x = self.hx.to("cuda", non_blocking=True)
        w = self.hw.to("cuda", non_blocking=True)
        qx, sx = f.fp8_quantize_act_1x128(x)
        qw, sw = f.fp8_quantize_weight_128x128(w, transpose_out=True)
        for h, d in ((self.hqx, qx), (self.hsx, sx), (self.hqw, qw), (self.hsw, sw)):
            h.copy_(d, non_blocking=True)

    def oracle_sample(self, orc, rows, nbs):
        x, w = synth.quant_inputs("cpu") if not hasattr(self, "_cpu") else self._cpu
        self._cpu = (x, w)
        xa = x[:rows * 8].contiguous().view(torch.int16).numpy().view(np.uint16)
        orc.quantize_act_1x128(xa)
        moved = xa.size * 3 + xa.shape[0] * (xa.shape[1] // 128) * 4
        blk = w[:, :nbs * 128].contiguous().view(torch.int16).numpy().view(np.uint16)
        orc.quantize_weight_128x128(blk, transpose_out=True)
        moved += blk.size * 3 + (blk.shape[0] // 128) * (blk.shape[1] // 128) * 4
        return float(moved)


class Dequant(Workload):
    """Codes back to bf16: the FFN weight W [7168 x 18432] quantized in 128x128
    blocks (untransposed), dequantized every step."""
    name = "dequant_w7168x18432_bf16"
    unit = "GB/s"
    dominant = "dequantize"
    sample_text = "%d rows x %d 128-column blocks of the codes, dequantized to bf16"

    def __init__(self, fp8, device, K=7168, N=18432):
        self.fp8, self.K, self.N = fp8, K, N
        self.kernels = ["dequantize"]
        if device is None:
            return
        w = synth.weight_input(K, N, 0.02, synth.FFN.config_id, device)
        self.q, self.s = fp8.fp8_quantize_weight_128x128(w, transpose_out=False)
        del w
        self.out = torch.empty((K, N), dtype=torch.bfloat16, device=device)

    def config(self):
        return {"workload": self.name, "codes": "E4M3 [%dx%d], 128x128 block scales" % (self.K, self.N),
                "out": "bf16", "source": "FFN W N(0,0.02) quantized once before timing",
                "l2": "codes 132 MB + output 264 MB > L2"}

    def algorithmic(self):
        K, N = self.K, self.N
        return {"dequantize": ("bytes", K * N * 3 + (K // 128) * (N // 128) * 4)}

    def work_per_step(self):
        return sum(v for _, v in self.algorithmic().values())

    def step(self, marks):
        marks(0)
        self.fp8.fp8_dequantize(self.q, self.s, 128, out=self.out)
        marks(1)

    def e2e_setup(self):
        self.hq = self.q.cpu().pin_memory()
        self.hs = self.s.cpu().pin_memory()
        self.hout = torch.empty((self.K, self.N), dtype=torch.bfloat16, pin_memory=True)
        return self.hq.numel() + self.hs.numel() * 4, self.hout.numel() * 2

    def e2e_step(self):
        q = self.hq.to("cuda", non_blocking=True)
        s = self.hs.to("cuda", non_blocking=True)
        self.hout.copy_(self.fp8.fp8_dequantize(q, s, 128), non_blocking=True)

    def oracle_sample(self, orc, rows, nbs):
        # codes of the first nbs column blocks (quantized once, untimed use
        # of the oracle's quantizer; re-made when a wider sample is asked for)
        if getattr(self, "_cpu_nbs", 0) < nbs:
            w = synth.weight_input(self.K, self.N, 0.02, synth.FFN.config_id, "cpu")
            blk = w[:, :nbs * 128].contiguous().view(torch.int16).numpy().view(np.uint16)
            self._cpu, self._cpu_nbs = orc.quantize_weight_128x128(blk), nbs
        q, s = self._cpu
        n = min(rows * 8, q.shape[0])
        qs = q[:n, :nbs * 128]
        out = orc.dequantize_fp32(qs, s[: (n + 127) // 128, :nbs], 128)
        orc.f32_to_bf16_bits(out)
        return float(qs.size * 3 + ((n + 127) // 128) * nbs * 4)


class DGrad(FFN):
    """dX = dY W^T with W quantized untransposed (K-major for this product)."""
    name = synth.DGRAD.name

    def __init__(self, fp8, device, M=16384, K=18432, N=7168):
        self.fp8, self.M, self.K, self.N = fp8, M, K, N
        self.kernels = ["quant_act_1x128", "quant_weight_128x128", "blockscaled_gemm"]
        if device is None:
            return
        self.x, self.w = synth.dgrad_inputs(device, M, K, N)    # dY [M,K], W [N,K]
        self.qx = torch.empty((M, K), dtype=torch.uint8, device=device)
        self.sx = torch.empty((M, K // 128), dtype=torch.float32, device=device)
        self.qw = torch.empty((N, K), dtype=torch.uint8, device=device)
        self.sw = torch.empty((N // 128, K // 128), dtype=torch.float32, device=device)
        self.c = torch.empty((M, N), dtype=torch.bfloat16, device=device)

    def config(self):
        return {"workload": self.name, "M": self.M, "N": self.N, "K": self.K,
                "dY": "bf16 [%dx%d] N(0,1e-3) 0.1%% outliers x100" % (self.M, self.K),
                "W": "bf16 [%dx%d] N(0,0.02), 128x128 blocks read transposed" % (self.N, self.K),
                "out": "bf16", "l2": "inputs larger than L2 (dY 604 MB)"}

    def algorithmic(self):
        M, N, K = self.M, self.N, self.K
        return {
            "quant_act_1x128": ("bytes", M * K * 2 + M * K + M * (K // 128) * 4),
            "quant_weight_128x128": ("bytes", K * N * 2 + K * N + (K // 128) * (N // 128) * 4),
            "blockscaled_gemm": ("flops", 2.0 * M * N * K),
        }

    def quant_error(self, rows=256, blocks=16):
        """dX = dY W^T on a sample of rows x 128-column blocks against the fp64
        product of the unquantized bf16 dY and W."""
        dev = self.c.device
        r = sample_index(self.M, rows, dev)
        nb = sample_index(self.N // 128, blocks, dev)
        cols = (nb[:, None] * 128 + torch.arange(128, device=dev)).reshape(-1)
        exact = self.x[r].double() @ self.w[cols].double().t()
        return error_vs_exact(self.c[r][:, cols].double(), exact,
                              "%d rows x %d 128-column blocks, spread evenly" % (len(r), len(nb)))

    def step(self, marks):
        f = self.fp8
        marks(0)
        f.fp8_quantize_act_1x128(self.x, q=self.qx, sa=self.sx)
        marks(1)
        f.fp8_quantize_weight_128x128(self.w, transpose_out=False, q=self.qw, sb=self.sw)
        marks(2)
        f.fp8_blockscaled_gemm(self.qx, self.sx, self.qw, self.sw, c=self.c, sb_kb_nb=False)
        marks(3)

    def e2e_setup(self):
        self.hx = self.x.cpu().pin_memory()
        self.hw = self.w.cpu().pin_memory()
        self.hc = torch.empty((self.M, self.N), dtype=torch.bfloat16, pin_memory=True)
        return (self.hx.numel() + self.hw.numel()) * 2, self.hc.numel() * 2

    def e2e_step(self):
        f = self.fp8
        x = self.hx.to("cuda", non_blocking=True)
        w = self.hw.to("cuda", non_blocking=True)
        qx, sx = f.fp8_quantize_act_1x128(x)
        qw, sw = f.fp8_quantize_weight_128x128(w, transpose_out=False)
        c = f.fp8_blockscaled_gemm(qx, sx, qw, sw, sb_kb_nb=False)
        self.hc.copy_(c, non_blocking=True)

    def oracle_sample(self, orc, rows, nbs):
        dy, w = synth.dgrad_inputs("cpu", self.M, self.K, self.N) if not hasattr(self, "_cpu") \
            else self._cpu
        self._cpu = (dy, w)
        xa = dy[:rows].contiguous().view(torch.int16).numpy().view(np.uint16)
        qa, sa = orc.quantize_act_1x128(xa)
        flops = 0.0
        for nb in range(nbs):
            blk = w[nb * 128:(nb + 1) * 128].contiguous().view(torch.int16).numpy().view(np.uint16)
            qb, sb = orc.quantize_weight_128x128(blk, transpose_out=False)
            orc.gemm_ref(qa, sa, qb, sb, b_kmajor=True, sb_transposed=True)
            flops += 2.0 * rows * 128 * self.K
        return flops


class WGrad(Workload):
    """dW = X^T dY: X and dY quantized in 1x128 tiles along the tokens (the
    contraction), written transposed; the GEMM with per-column B scales."""
    name = synth.WGRAD.name
    unit = "TFLOP/s"
    dominant = "blockscaled_gemm_colscale"
    sample_text = ("%d rows x %d 128-column blocks of dW, with the 128x1 quantization of the "
                   "X and dY columns they use")

    def __init__(self, fp8, device, M=16384, K=7168, N=18432):
        self.fp8, self.M, self.K, self.N = fp8, M, K, N
        self.kernels = ["quant_act_128x1_x", "quant_act_128x1_dy", "blockscaled_gemm_colscale"]
        if device is None:
            return
        self.x, self.dy = synth.wgrad_inputs(device, M, K, N)      # [M, K], [M, N]
        self.qxt = torch.empty((K, M), dtype=torch.uint8, device=device)
        self.sxt = torch.empty((K, M // 128), dtype=torch.float32, device=device)
        self.qdt = torch.empty((N, M), dtype=torch.uint8, device=device)
        self.sdt = torch.empty((M // 128, N), dtype=torch.float32, device=device)
        self.c = torch.empty((K, N), dtype=torch.float32, device=device)

    def config(self):
        return {"workload": self.name, "tokens": self.M, "K": self.K, "N": self.N,
                "x": "bf16 [%dx%d] N(0,1) 0.1%% outliers x100" % (self.M, self.K),
                "dy": "bf16 [%dx%d] N(0,1e-3) 0.1%% outliers x100" % (self.M, self.N),
                "out": "fp32 dW [%dx%d]" % (self.K, self.N),
                "l2": "inputs larger than L2 (X+dY bf16 = %.0f MB > 126 MB)" %
                      ((self.M * self.K + self.M * self.N) * 2 / 1e6)}

    def flops(self):
        return 2.0 * self.M * self.N * self.K

    def work_per_step(self):
        return self.flops()

    def algorithmic(self):
        M, N, K = self.M, self.N, self.K
        return {
            "quant_act_128x1_x": ("bytes", M * K * 2 + M * K + (M // 128) * K * 4),
            "quant_act_128x1_dy": ("bytes", M * N * 2 + M * N + (M // 128) * N * 4),
            "blockscaled_gemm_colscale": ("flops", 2.0 * M * N * K),
        }

    def quant_error(self, rows=256, blocks=16):
        """dW = X^T dY on a sample of rows x 128-column blocks against the fp64
        product of the unquantized bf16 X and dY (contraction over all tokens)."""
        dev = self.c.device
        r = sample_index(self.K, rows, dev)
        nb = sample_index(self.N // 128, blocks, dev)
        cols = (nb[:, None] * 128 + torch.arange(128, device=dev)).reshape(-1)
        exact = self.x[:, r].double().t() @ self.dy[:, cols].double()
        return error_vs_exact(self.c[r][:, cols].double(), exact,
                              "%d rows x %d 128-column blocks, spread evenly" % (len(r), len(nb)))

    def step(self, marks):
        f = self.fp8
        marks(0)
        f.fp8_quantize_act_128x1(self.x, qt=self.qxt, st=self.sxt)
        marks(1)
        f.fp8_quantize_act_128x1(self.dy, qt=self.qdt, st=self.sdt, st_kb_major=True)
        marks(2)
        f.fp8_blockscaled_gemm_colscale(self.qxt, self.sxt, self.qdt, self.sdt, c=self.c)
        marks(3)

    def e2e_setup(self):
        self.hx = self.x.cpu().pin_memory()
        self.hdy = self.dy.cpu().pin_memory()
        self.hc = torch.empty((self.K, self.N), dtype=torch.float32, pin_memory=True)
        return (self.hx.numel() + self.hdy.numel()) * 2, self.hc.numel() * 4

    def e2e_step(self):
        x = self.hx.to("cuda", non_blocking=True)
        dy = self.hdy.to("cuda", non_blocking=True)
        self.hc.copy_(self.fp8.linear_weight_grad(x, dy), non_blocking=True)

    def oracle_sample(self, orc, rows, nbs):
        """dW rows 0..rows-1 (columns of X) x the first nbs 128-column blocks
        (columns of dY), each column quantized 128x1 over all tokens."""
        if not hasattr(self, "_cpu"):
            self._cpu = synth.wgrad_inputs("cpu", self.M, self.K, self.N)
        x, dy = self._cpu
        xa = x[:, :rows].contiguous().view(torch.int16).numpy().view(np.uint16)
        qa, sa = orc.quantize_act_128x1(xa)
        flops = 0.0
        for nb in range(nbs):
            blk = dy[:, nb * 128:(nb + 1) * 128].contiguous().view(torch.int16).numpy() \
                .view(np.uint16)
            qb, sb = orc.quantize_act_128x1(blk)
            orc.gemm_ref_colscale(qa, sa, qb, sb)
            flops += 2.0 * rows * 128 * self.M
        return flops


class MoE(Workload):
    name = synth.MOE.name
    unit = "TFLOP/s"
    dominant = "grouped_gemm_gate_up"

    def __init__(self, fp8, device, tokens=8192, experts=256, topk=8, hidden=7168, inter=2048,
                 dispatch="scatter"):
        self.fp8 = fp8
        self.T, self.E, self.k, self.H, self.I = tokens, experts, topk, hidden, inter
        self.R = tokens * topk
        # the dispatch in row order (gather: output row r <- token rows[r]) or
        # in token order (scatter: token t -> rows dest[t, :])
        self.dispatch = dispatch
        self.dispatch_kernel = "quant_act_1x128_%s_x" % dispatch
        self.kernels = [self.dispatch_kernel, "grouped_gemm_gate_up", "quant_act_1x128_h",
                        "grouped_gemm_down"]
        if device is None:
            return
        d = synth.moe_inputs(device, tokens, experts, topk, hidden, inter, with_weights=False)
        # tokens and their routing: the dispatch (token rows to expert order) is
        # fused into the activation quantizer
        self.x, self.h, self.off = d["x"], d["h_down"], d["offsets"]
        self.rows = d["token_of"].to(torch.int32)
        # the same routing in token order: token t's topk expert-sorted rows
        self.dest = synth.moe_dispatch_dest(d["token_of"], tokens, topk)
        del d
        R, H, I, E = self.R, hidden, inter, experts
        self.qgu = torch.empty((E, 2 * I, H), dtype=torch.uint8, device=device)
        self.sgu = torch.empty((E, H // 128, 2 * I // 128), dtype=torch.float32, device=device)
        self.qdn = torch.empty((E, H, I), dtype=torch.uint8, device=device)
        self.sdn = torch.empty((E, I // 128, H // 128), dtype=torch.float32, device=device)
        for e in range(E):   # expert weights: quantized once, outside the timed region
            w = synth.moe_expert_weight(e, "gate_up", device, hidden, inter)
            fp8.fp8_quantize_weight_128x128(w, transpose_out=True, q=self.qgu[e], sb=self.sgu[e])
            w = synth.moe_expert_weight(e, "down", device, hidden, inter)
            fp8.fp8_quantize_weight_128x128(w, transpose_out=True, q=self.qdn[e], sb=self.sdn[e])
        del w
        self.qx = torch.empty((R, H), dtype=torch.uint8, device=device)
        self.sx = torch.empty((R, H // 128), dtype=torch.float32, device=device)
        self.qh = torch.empty((R, I), dtype=torch.uint8, device=device)
        self.sh = torch.empty((R, I // 128), dtype=torch.float32, device=device)
        self.cgu = torch.empty((R, 2 * I), dtype=torch.bfloat16, device=device)
        self.cdn = torch.empty((R, H), dtype=torch.bfloat16, device=device)
        torch.cuda.synchronize()

    def config(self):
        return {"workload": self.name, "tokens": self.T, "experts": self.E, "topk": self.k,
                "routed_rows": self.R, "gate_up": "K=%d N=%d" % (self.H, 2 * self.I),
                "down": "K=%d N=%d" % (self.I, self.H), "out": "bf16",
                "weights": "quantized once before timing (11.27 GB E4M3)",
                "dispatch": ("routed rows gathered from the token rows inside the activation "
                             "quantizer" if self.dispatch == "gather" else
                             "each token row quantized once inside the activation quantizer and "
                             "written to its 8 expert-sorted rows"),
                "l2": "expert weights 11.27 GB >> L2"}

    def algorithmic(self):
        R, H, I, E = self.R, self.H, self.I, self.E
        return {
            # tokens read once, routed rows written (codes + scales)
            self.dispatch_kernel: ("bytes", self.T * H * 2 + R * H + R * (H // 128) * 4),
            "grouped_gemm_gate_up": ("flops", 2.0 * R * 2 * I * H),
            "quant_act_1x128_h": ("bytes", R * I * 3 + R * (I // 128) * 4),
            "grouped_gemm_down": ("flops", 2.0 * R * H * I),
        }

    def hbm_bytes(self, kernel):
        R, H, I, E = self.R, self.H, self.I, self.E
        if kernel == "grouped_gemm_gate_up":
            return E * 2 * I * H + R * H + R * 2 * I * 2
        if kernel == "grouped_gemm_down":
            return E * H * I + R * I + R * H * 2
        return None

    def work_per_step(self):
        return 2.0 * self.R * 2 * self.I * self.H + 2.0 * self.R * self.H * self.I

    def quant_error(self, rows=64, blocks=16, experts=4):
        """Both grouped GEMMs of the last step on a sample (experts spread over
        the range, rows spread within each expert, 128-column blocks spread
        over N) against the fp64 products of the unquantized bf16 inputs and
        that expert's bf16 weights."""
        dev = self.cgu.device
        off = self.off.cpu().tolist()
        out = {}
        for which, a, c, N in (("gate_up", None, self.cgu, 2 * self.I),
                                  ("down", self.h, self.cdn, self.H)):
            got, exact = [], []
            nb = sample_index(N // 128, blocks, dev)
            cols = (nb[:, None] * 128 + torch.arange(128, device=dev)).reshape(-1)
            for e in sample_index(self.E, experts, "cpu").tolist():
                lo, hi = off[e], off[e + 1]
                if hi <= lo:
                    continue
                r = lo + sample_index(hi - lo, rows, dev)
                w = synth.moe_expert_weight(e, which, dev, self.H, self.I)[:, cols].double()
                src = self.x[self.rows[r].long()] if a is None else a[r]
                exact.append(src.double() @ w)
                got.append(c[r][:, cols].double())
            out[which] = error_vs_exact(torch.cat(got), torch.cat(exact),
                                        "%d experts x up to %d rows x %d 128-column blocks"
                                        % (experts, rows, len(nb)))
        return out

    def launches_per_step(self):
        # a grouped GEMM of K >= 4096 is two launches: CTA-pair tiles, then
        # the groups' 1-128-row remainders on the one-CTA kernel
        return len(self.kernels) + (self.H >= 4096) + (self.I >= 4096)

    def step(self, marks):
        f = self.fp8
        marks(0)
        if self.dispatch == "gather":
            f.fp8_quantize_act_1x128_gather(self.x, self.rows, q=self.qx, sa=self.sx)
        else:
            f.fp8_quantize_act_1x128_scatter(self.x, self.dest, self.R, q=self.qx, sa=self.sx)
        marks(1)
        f.fp8_grouped_gemm(self.qx, self.sx, self.qgu, self.sgu, self.off, c=self.cgu)
        marks(2)
        f.fp8_quantize_act_1x128(self.h, q=self.qh, sa=self.sh)
        marks(3)
        f.fp8_grouped_gemm(self.qh, self.sh, self.qdn, self.sdn, self.off, c=self.cdn)
        marks(4)

    def e2e_setup(self):
        self.hx = self.x.cpu().pin_memory()
        self.hrows = self.rows.cpu().pin_memory()
        self.hdest = self.dest.cpu().pin_memory()
        self.hh = self.h.cpu().pin_memory()
        self.hoff = self.off.cpu().pin_memory()
        self.hgu = torch.empty_like(self.cgu, device="cpu").pin_memory()
        self.hdn = torch.empty_like(self.cdn, device="cpu").pin_memory()
        route = self.hrows if self.dispatch == "gather" else self.hdest
        return ((self.hx.numel() + self.hh.numel()) * 2 + (self.hoff.numel() + route.numel()) * 4,
                (self.hgu.numel() + self.hdn.numel()) * 2)

    def e2e_step(self):
        f = self.fp8
        x = self.hx.to("cuda", non_blocking=True)
        h = self.hh.to("cuda", non_blocking=True)
        off = self.hoff.to("cuda", non_blocking=True)
        if self.dispatch == "gather":
            qx, sx = f.fp8_quantize_act_1x128_gather(x, self.hrows.to("cuda", non_blocking=True))
        else:
            qx, sx = f.fp8_quantize_act_1x128_scatter(x, self.hdest.to("cuda", non_blocking=True),
                                                      self.R)
        cgu = f.fp8_grouped_gemm(qx, sx, self.qgu, self.sgu, off)
        qh, sh = f.fp8_quantize_act_1x128(h)
        cdn = f.fp8_grouped_gemm(qh, sh, self.qdn, self.sdn, off)
        self.hgu.copy_(cgu, non_blocking=True)
        self.hdn.copy_(cdn, non_blocking=True)

    def oracle_sample(self, orc, rows, nbs):
        """Expert 0's first `rows` routed rows x `nbs` column blocks of both GEMMs."""
        if not hasattr(self, "_cpu"):
            d = synth.moe_inputs("cpu", self.T, self.E, self.k, self.H, self.I, with_weights=False)
            self._cpu = (d, synth.moe_expert_weight(0, "gate_up", "cpu", self.H, self.I),
                         synth.moe_expert_weight(0, "down", "cpu", self.H, self.I))
        d, wgu, wdn = self._cpu
        flops = 0.0
        for a, w, K in ((d["x_routed"], wgu, self.H), (d["h_down"], wdn, self.I)):
            xa = a[:rows].contiguous().view(torch.int16).numpy().view(np.uint16)
            qa, sa = orc.quantize_act_1x128(xa)
            for nb in range(nbs):
                blk = w[:, nb * 128:(nb + 1) * 128].contiguous().view(torch.int16).numpy() \
                    .view(np.uint16)
                qb, sb = orc.quantize_weight_128x128(blk, transpose_out=True)
                orc.gemm_ref(qa, sa, qb, sb)
                flops += 2.0 * rows * 128 * K
        return flops


WORKLOADS = {"ffn": FFN, "ffn_q": FFNQuantOut, "quant": Quant, "moe": MoE, "dgrad": DGrad,
             "dequant": Dequant, "wgrad": WGrad}
# Reported with the default run, after the FFN headline, each in its own timed region.
EXTRA_WORKLOADS = ("quant", "dgrad", "wgrad", "moe", "ffn_q", "dequant")
# Oracle sample per step of the reference arm: (rows, column blocks).  Each is
# about 60% of the CPU-baseline sample below, with the same balance of
# quantization and GEMM work (so that both arms measure the oracle alike),
# and a 25-step run stays within a few minutes.
ORACLE_SAMPLE = {"ffn": (768, 32), "ffn_q": (768, 32), "quant": (256, 144), "moe": (256, 24),
                 "dgrad": (256, 14), "dequant": (512, 144), "wgrad": (256, 24)}
# The single CPU-baseline measurement of a run: about 10 s of oracle work.
CPU_BASELINE_SAMPLE = {"ffn": (1024, 60), "ffn_q": (1024, 60), "quant": (512, 144),
                       "moe": (512, 24), "dgrad": (256, 24), "dequant": (896, 144),
                       "wgrad": (512, 24)}


# ----------------------------------------------------------------------------- timing

def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank contributes its own device-timed
    milliseconds and all of them get the maximum (one collective, taken in
    the same order on every rank)."""
    if world <= 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world, work_per_step, steps, max_ms):
    """Whole-job throughput of `world` replicas that each did `steps` steps
    of `work_per_step` units, timed as the slowest rank (weak scaling)."""
    return world * work_per_step * steps / (max_ms / 1e3)


def make_workload(args, fp8, device):
    """The workload object; --moe-experts E shrinks the MoE workload to E
    experts and 32 E tokens (same rows per expert), for profiler captures
    that must stay small."""
    if args.workload == "moe":
        return MoE(fp8, device, tokens=32 * args.moe_experts, experts=args.moe_experts,
                   dispatch=args.moe_dispatch)
    return WORKLOADS[args.workload](fp8, device)


def time_workload(wl, args, world, device, fp8):
    """W untimed warm-up steps, then exactly K steps between barriers and
    device synchronizations, timed with CUDA events on the launching stream
    (whole region and each kernel of each step); SM clocks sampled during the
    timed region.  Returns (max-over-ranks ms, per-kernel mean ms, clocks,
    wall seconds, device error word)."""
    stream = torch.cuda.current_stream()
    nk = len(wl.kernels)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        wl.step(lambda i: None)
    torch.cuda.synchronize()
    if fp8.fp8_get_device_error() != 0:
        raise RuntimeError("device error during warm-up of %s" % wl.name)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    time.sleep(0.3)
    clocks.begin()
    wall0 = time.perf_counter()
    # A short device-side spin, enqueued before the start event, keeps the
    # GPU busy while the host enqueues the first step's launches: the region
    # then holds the steps' GPU work, not the host's first-launch latency
    # after the synchronize above (which had inflated the first kernel of
    # step 0, and so its per-kernel mean, by tens of microseconds).
    torch.cuda._sleep(QUEUE_FILL_CYCLES)
    start.record(stream)
    for s in range(args.steps):
        wl.step(lambda i, s=s: ev[s][i].record(stream))
    stop.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world, device)
    dev_err = fp8.fp8_get_device_error()
    per_kernel = {}
    for i, k in enumerate(wl.kernels):
        per_kernel[k] = statistics.fmean(ev[s][i].elapsed_time(ev[s][i + 1])
                                         for s in range(args.steps))
    return elapsed_ms, per_kernel, clk, wall, dev_err


def run_ours(args, rank, world, local_rank):
    import fp8_fine_grained_online_b200 as fp8
    device = "cuda:%d" % local_rank
    torch.cuda.set_device(local_rank)
    wl = make_workload(args, fp8, device)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    elapsed_ms, per_kernel, clk, wall, dev_err = time_workload(wl, args, world, device, fp8)

    # end to end through the public API, pinned host buffers
    e2e = None
    if not args.no_e2e:
        h2d, d2h = wl.e2e_setup()
        wl.e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(1, args.steps)   # the same K steps as the device-timed region
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_e2e):
            wl.e2e_step()
        wl.e2e_join(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        e2e = {"value": round(aggregate_rate(world, wl.work_per_step(), n_e2e, e_ms) / scale(wl), 3),
               "unit": wl.unit, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e}
        wl.e2e_teardown()
    return wl, elapsed_ms, per_kernel, clk, e2e, wall, dev_err


def run_extra(args, name, world, local_rank, peaks, peak_src):
    """One more workload on the same process (every rank, as for the
    headline): its own timed region, kernels, roofline and clocks."""
    import fp8_fine_grained_online_b200 as fp8
    device = "cuda:%d" % local_rank
    wl = WORKLOADS[name](fp8, device)
    elapsed_ms, per_kernel, clk, wall, dev_err = time_workload(wl, args, world, device, fp8)
    rec = workload_record(wl, name, world, args, elapsed_ms, per_kernel, peaks, peak_src)
    rec.update({"clocks": clk, "device_error": dev_err, "wall_s_timed_region": round(wall, 4)})
    err = wl.quant_error() if callable(getattr(wl, "quant_error", None)) else None
    del wl
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec, err


def workload_record(wl, name, world, args, elapsed_ms, per_kernel, peaks, peak_src):
    value = aggregate_rate(world, wl.work_per_step(), args.steps, elapsed_ms) / scale(wl)
    kernels = {}
    for k, ms in per_kernel.items():
        r = roofline_entry(wl, k, ms, peaks, peak_src)
        kernels[k] = {"us": round(ms * 1e3, 2), "achieved": r["achieved"], "unit": r["unit"],
                      "frac": r["frac"], "bound": r["bound"],
                      "traffic": recorded_traffic(k, name)}
    roof = roofline_entry(wl, wl.dominant, per_kernel[wl.dominant], peaks, peak_src)
    roof["traffic"] = recorded_traffic(wl.dominant, name)
    return {"config": wl.config(), "value": round(value, 3), "unit": wl.unit,
            "ms_per_step": round(elapsed_ms / args.steps, 4), "steps": args.steps,
            "warmup": args.warmup, "gpu_launches": wl.launches_per_step() * args.steps,
            "roofline": roof, "kernels": kernels}


def scale(wl):
    return 1e12 if wl.unit == "TFLOP/s" else 1e9


def roofline_entry(wl, kernel, ms, peaks, peak_src):
    kind, amount = wl.algorithmic()[kernel]
    if kind == "flops" and wl.unit == "TFLOP/s" and hasattr(wl, "hbm_bytes") \
            and wl.hbm_bytes(kernel) is not None:
        # grouped GEMM: weight streaming; report the bound that limits it
        t_flop = amount / (peaks["bf16_tflops"] * FP8_OVER_BF16 * 1e12)
        t_hbm = wl.hbm_bytes(kernel) / (peaks["hbm_gbs"] * 1e9)
        if t_hbm > t_flop:
            ach = wl.hbm_bytes(kernel) / (ms / 1e3) / 1e9
            return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                    "basis": "HBM bytes of fp8 weights + act + out per launch, %s copy peak" %
                             peak_src}
    if kind == "flops":
        peak = peaks["bf16_tflops"] * FP8_OVER_BF16
        ach = amount / (ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": round(ach, 1), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                "basis": "%s bf16 burst x 2 (fp8/bf16 nominal dense ratio)" % peak_src}
    ach = amount / (ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4), "basis": "%s copy peak" % peak_src}


def cpu_baseline(args, wl_cls):
    import oracle
    wl = wl_cls(None, None)
    rows, nbs = CPU_BASELINE_SAMPLE[args.workload]
    wl.oracle_sample(oracle, 1, nbs)            # input generation + library load, untimed
    t0 = time.perf_counter()
    work = wl.oracle_sample(oracle, rows, nbs)
    dt = time.perf_counter() - t0
    return {"value": round(work / dt / scale(wl), 6), "unit": wl.unit,
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": getattr(wl, "sample_text", "%d rows x %d 128-column blocks of the step, "
                              "with their online quantization") % (rows, nbs) + " (%.1f s)" % dt}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="ffn")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra", default=None,
                    help="comma list of workloads timed after the headline and reported under "
                         "'workloads' (default: all others when the headline is ffn; 'none')")
    ap.add_argument("--no-quant-error", action="store_true")
    ap.add_argument("--moe-dispatch", choices=["gather", "scatter"], default="scatter",
                    help="MoE workload only: dispatch in row order (gather) or token order")
    ap.add_argument("--moe-experts", type=int, default=256,
                    help="MoE workload only: number of experts (tokens = 32 x experts)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl_cls = WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return
        import oracle
        wl = wl_cls(None, None)
        rows, nbs = ORACLE_SAMPLE[args.workload]
        wl.oracle_sample(oracle, 1, nbs)
        for _ in range(args.warmup):
            wl.oracle_sample(oracle, 2, nbs)
        t0 = time.perf_counter()
        work = 0.0
        for _ in range(args.steps):
            work += wl.oracle_sample(oracle, rows, nbs)
        dt = time.perf_counter() - t0
        v = round(work / dt / scale(wl), 6)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": v, "unit": wl.unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": wl.config(),
            "cpu_baseline": {"value": v, "unit": wl.unit, "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": "per step: %d rows x %d 128-column blocks of the "
                                       "workload with their online quantization" % (rows, nbs)},
            "e2e": {"value": v, "unit": wl.unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }))
        return

    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    extras = parse_extra(args)
    try:
        import fp8_fine_grained_online_b200 as fp8
        wl, elapsed_ms, per_kernel, clk, e2e, wall, dev_err = run_ours(args, rank, world,
                                                                       local_rank)
        peaks, peak_src = load_peaks()
        # Quantization error of the FP8 path against the unquantized fp64
        # product: the tiny config in full, the headline on a sample.
        errors = {}
        if not args.no_quant_error:
            errors["tiny"] = quant_error_tiny(fp8, "cuda:%d" % local_rank)
            if callable(getattr(wl, "quant_error", None)):
                errors[args.workload] = wl.quant_error()
        head = workload_record(wl, args.workload, world, args, elapsed_ms, per_kernel, peaks,
                               peak_src)
        del wl
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        # The other configurations, each timed in its own region like the
        # headline (its own warm-up, steps, clocks and roofline).
        others = {}
        for name in extras:
            rec, err = run_extra(args, name, world, local_rank, peaks, peak_src)
            others[name] = rec
            if err is not None and not args.no_quant_error:
                errors[name] = err
        if rank != 0:
            return
        line = {
            "metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 (fp32 accumulate)",
            "data": "synthetic (seeded, DeepSeek-V3 layer shapes)", "config": head["config"],
            "roofline": head["roofline"], "kernels": head["kernels"],
            "gpu_launches": head["gpu_launches"],
            "clocks": clk, "e2e": e2e, "device_error": dev_err,
            "wall_s_timed_region": round(wall, 4),
            "parallelism": "replicas (dp%d, no collective on the data path)" % world,
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                      "source": peak_src},
        }
        if errors:
            line["quant_error"] = {
                "reference": "fp64 product of the unquantized inputs (C_exact)",
                "metrics": "max_rel = max|C - C_exact| / max|C_exact|; "
                           "fro_rel = ||C - C_exact||_F / ||C_exact||_F",
                **errors}
        if others:
            line["workloads"] = others
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args, wl_cls)
        print(json.dumps(line))
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


def parse_extra(args):
    """Workloads timed after the headline: by default every other
    configuration when the headline is the FFN forward, none otherwise."""
    if args.extra is None:
        return list(EXTRA_WORKLOADS) if args.workload == "ffn" else []
    if args.extra == "none":
        return []
    names = [n for n in args.extra.split(",") if n]
    for n in names:
        if n not in WORKLOADS:
            raise SystemExit("unknown workload in --extra: %s" % n)
    return [n for n in names if n != args.workload]

if __name__ == "__main__":
    main()
