"""Seeded synthetic inputs for the SparsePR attention call.

This package only draws random numbers and names workload shapes. It holds no
step of the attention method, so both the CPU oracle and the CUDA path can use
it without sharing any of the method's arithmetic.
"""
from .workloads import WORKLOADS, Workload, get_workload
from .generator import video_qkv, video_qkv_device, bf16_bits_from_f32, bf16_bits_to_f32, bf16_bits_to_f64

__all__ = [
    "WORKLOADS",
    "Workload",
    "get_workload",
    "video_qkv",
    "video_qkv_device",
    "bf16_bits_from_f32",
    "bf16_bits_to_f32",
    "bf16_bits_to_f64",
]
