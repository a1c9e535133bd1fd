"""Host-side helpers of bench.py that need no GPU: the clock summary's choice of
samples, and the PCI bus id it filters on."""
import types

import bench


def _sample(t, mhz, reasons=("Not Active",) * 4, start=None):
    s = (t, float(mhz), 1965.0, list(reasons))
    return s if start is None else s + (start,)


def test_clock_summary_counts_queries_that_overlap_the_region():
    c = bench.ClockSampler(None)
    # an nvidia-smi sample long before, an NVML query that started before the region and
    # ended inside it, and one that started after the region ended
    c.samples = [_sample(9.0, 1000), _sample(10.0012, 1965, start=10.0002),
                 _sample(10.0030, 1800, start=10.0025)]
    s = c.summary(10.0005, 10.0020, 10.5)
    assert s["samples_in_timed_region"] == 1 and s["sm_mhz"] == 1965.0
    assert s["window"].startswith("the timed region")


def test_clock_summary_falls_back_to_the_surrounding_window():
    c = bench.ClockSampler(None)
    c.samples = [_sample(9.95, 1965, reasons=("Not Active",) * 3 + ("Active",)),
                 _sample(10.40, 1950)]
    s = c.summary(10.0005, 10.0020, 10.3)
    assert s["samples_in_timed_region"] == 0 and s["samples"] == 2
    assert s["reasons"] == ["sw_power_cap"] and s["sm_mhz"] == 1957.5


def test_clock_summary_without_samples():
    s = bench.ClockSampler(None).summary(1.0, 2.0)
    assert s["samples"] == 0 and s["sm_mhz"] is None


def test_bus_id_format():
    props = types.SimpleNamespace(pci_bus_id=0x1B, pci_domain_id=0, pci_device_id=0)
    fake = types.SimpleNamespace(cuda=types.SimpleNamespace(get_device_properties=lambda d: props))
    assert bench.bus_id_of(fake, 0) == "00000000:1b:00.0"
    none = types.SimpleNamespace(cuda=types.SimpleNamespace(
        get_device_properties=lambda d: types.SimpleNamespace()))
    assert bench.bus_id_of(none, 0) is None
